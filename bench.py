"""Benchmark of MLA decoding over a paged latent KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole decode path over one batch of synthetic input:
the split-KV planner, the decode kernel (page fetch, QK, online softmax, PV,
finalize) and the split-combine kernel (for the fused workload also the
RMSNorm/RoPE prologue and the conjugate-RoPE/FP8 epilogue; for the sparse
workloads the FP8 gather/dequant).  Inputs are resident in HBM before the timed
region; every workload's KV cache is larger than the 126 MB L2, so no L2 flush
is inserted between steps.

Rank 0 prints ONE JSON line.  Multi-GPU runs are independent replicas (the
decode path has no exchange step): each rank decodes its own batch and
`value` aggregates all ranks' work over the slowest rank's time.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_paged_kv_03_b200 import workloads as W  # noqa: E402

METRIC = "MLA decode TFLOPS & KV-read GB/s on 1 B200, % of roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOAD_INFO = {
    "compute": ("Compute-bound dense decode, bf16: batch 64, s_q 1, h_q 128, d_qk 576, d_v 512, "
                "L ~ U[4096, 8192], block 64, shuffled blocks, q,k ~ 0.5 N(0,1)", "tensor"),
    "memory": ("Memory-bound dense decode, bf16: batch 128, s_q 2 (causal pair), h_q 16, d_qk 576, "
               "d_v 512, L log-uniform [1024, 16384], block 64, shuffled blocks", "hbm"),
    "fused": ("Fused RMSNorm-RoPE-attn-conjRoPE-FP8 decode: batch 32, s_q 1, h_q 64, d 576, d_v 576, "
              "L ~ U[2048, 32768], block 64", "hbm"),
    "fused_b1": ("Fused RMSNorm-RoPE-attn-conjRoPE-FP8 decode: batch 1, s_q 1, h_q 64, d 576, "
                 "d_v 576, L ~ U[2048, 32768], block 64", "hbm"),
    "sparse_v41": ("Token-level sparse decode, V4.1 FP8 528-byte cache (512 e4m3 + 16 e8m0): "
                   "batch 32, s_q 1, h_q 128, d_qk = d_v 512, 65536-token cache per sequence, "
                   "topk 2048, 5% -1 slots", "tensor"),
    "sparse_v41_fp4": ("Token-level sparse decode, V4.1 FP4 288-byte cache (512 e2m1 + 32 e4m3): "
                       "batch 32, s_q 1, h_q 128, d_qk = d_v 512, 65536-token cache per sequence, "
                       "topk 2048, 5% -1 slots", "tensor"),
    "fused_sparse": ("Fused RMSNorm-RoPE-attn-conjRoPE-FP8 decode in sparse mode over the FP8 "
                     "656-byte cache: batch 32, s_q 1, h_q 64, d 576, d_v 576, 65536-token cache "
                     "per sequence, topk 2048, 5% -1 slots, position L - 1", "tensor"),
    "sparse_prefill": ("Token-level sparse prefill, bf16 latent KV, no batch dimension: s_q 4096 "
                       "query tokens x h_q 128 over s_kv 4096 positions, topk 2048 rows at or "
                       "before each token, per-token top-k length, one sink per head, d_qk 576, "
                       "d_v 512", "tensor"),
    "sparse": ("Token-level sparse decode, FP8 656-byte cache: batch 32, s_q 1, h_q 128, d_v 512, "
               "65536-token cache per sequence, topk 2048, 5% -1 slots", "tensor"),
    "tiny": ("Tiny dense decode, bf16: batch 2, s_q 1, h_q 16, lengths {37, 200}", "tensor"),
}


# Sources each workload's dominant (attention) kernel is built from, with the
# launch code: its stored ncu traffic stays valid while these are unchanged.
_KERNEL_SOURCES = {
    "mla_pair_decode_kernel": ["pair_kernel.cuh", "decode_kernel.cuh"],
    "mla_page_decode_kernel": ["page_kernel.cuh", "decode_kernel.cuh"],
    "mla_decode_kernel": ["decode_kernel.cuh"],
}
_COMMON_SOURCES = ["ptx.cuh", "mla_common.h", "mla_api.cu"]


def kernel_source_hash(kernel="mla_decode_kernel"):
    """Hash of the CUDA sources of one kernel (its headers, the shared PTX and
    constant headers, and the launch code); a stored ncu traffic figure is
    used only while they are unchanged since it was captured."""
    import hashlib
    d = os.path.join(ROOT, "mla_paged_kv_03_b200", "csrc")
    key = next((k for k in _KERNEL_SOURCES if kernel.startswith(k)), None)
    names = sorted(_KERNEL_SOURCES[key] + _COMMON_SOURCES) if key else \
        sorted(n for n in os.listdir(d) if n.endswith((".cu", ".cuh", ".h")))
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def load_traffic(workload):
    """dram bytes read + written per launch of the attention kernel from the
    committed ncu summary, or None if absent or taken on other sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("source_hash") == kernel_source_hash(e.get("kernel", "")):
            return e["bytes_per_launch"]
    except Exception:
        pass
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ------------------------------------------------------------ work counting

def dense_work(case):
    """Algorithmic FLOPs and bytes: 2*|T|*(576 + d_v) per query row over its
    visible tokens; bytes = the latent rows read once per sequence (all rows
    share one KV head) + q + O + LSE + block table + lengths."""
    sl = case.cache_seqlens.cpu().tolist()
    flops = 0
    kv_tokens = 0
    for L in sl:
        for i in range(case.s_q):
            vis = max(0, min(L, L - case.s_q + 1 + i)) if case.causal else L
            flops += 2 * vis * (576 + case.d_v) * case.h_q
        kv_tokens += L
    kv_bytes = kv_tokens * 576 * 2
    io = case.q.numel() * 2 + case.batch * case.s_q * case.h_q * (case.d_v * 2 + 4) + \
        case.block_table.numel() * 4 + case.batch * 4
    return flops, kv_bytes, kv_bytes + io


def fused_work(case):
    sl = case.cache_seqlens.cpu().tolist()
    flops = sum(2 * L * (576 + 576) * case.h_q for L in sl)
    kv_bytes = sum(sl) * 576 * 2
    io = case.q_raw.numel() * 2 + 576 * 4 + case.batch * case.h_q * (576 + 4 + 4) + \
        case.block_table.numel() * 4 + case.batch * 4
    return flops, kv_bytes, kv_bytes + io


def fused_sparse_work(case):
    valid = int((case.indices >= 0).sum())  # sequences x valid slots (s_q = 1)
    flops = 2 * valid * (576 + 576) * case.h_q
    kv_bytes = valid * 656
    io = case.q_raw.numel() * 2 + 576 * 4 + case.indices.numel() * 4 + case.batch * 4 + \
        case.batch * case.h_q * (576 + 4 + 4)
    return flops, kv_bytes, kv_bytes + io


def prefill_work(case):
    n = case.topk_length.cpu().clamp(0, case.topk) if case.topk_length is not None else None
    ix = case.indices.cpu()
    if n is not None:
        ix = torch.where(torch.arange(case.topk)[None, :] < n[:, None], ix, torch.full_like(ix, -1))
    valid = int((ix >= 0).sum())  # (token, row) pairs
    flops = 2 * valid * (576 + case.d_v) * case.h_q
    kv_bytes = valid * 1152
    io = case.q.numel() * 2 + case.indices.numel() * 4 + case.s_q * case.h_q * (case.d_v * 2 + 4)
    return flops, kv_bytes, kv_bytes + io


def sparse_dims(case):
    """(latent width of q . k, bytes per cache row) of a sparse case."""
    row = int(case.kcache.shape[-1])
    return (576 if row == 656 else 512), row


def sparse_work(case):
    valid = int((case.indices >= 0).sum())  # (b, s_q) pairs x valid slots
    d_qk, row_bytes = sparse_dims(case)
    flops = 2 * valid * (d_qk + case.d_v) * case.h_q
    kv_bytes = valid * row_bytes
    io = case.q.numel() * 2 + case.indices.numel() * 4 + \
        case.batch * case.s_q * case.h_q * (case.d_v * 2 + 4)
    return flops, kv_bytes, kv_bytes + io


# ----------------------------------------------------------------- GPU arm

class GpuStep:
    """One decode step through the library's public API, inputs resident."""

    def __init__(self, name, seed, dev):
        from mla_paged_kv_03_b200 import binding as B
        self.B = B
        self.name = name
        self.dev = dev
        if name in ("compute", "memory", "tiny"):
            self.case = W.WORKLOADS[name](seed=seed, device=dev)
            self.kind = "dense"
            self.work = dense_work(self.case)
            c = self.case
            self.R = c.s_q * c.h_q
        elif name in ("fused", "fused_b1"):
            self.case = W.fused(seed=seed, device=dev, batch=32 if name == "fused" else 1)
            self.kind = "fused"
            self.work = fused_work(self.case)
            self.R = self.case.h_q
        elif name == "fused_sparse":
            self.case = W.fused_sparse(seed=seed, device=dev)
            self.kind = "fused_sparse"
            self.work = fused_sparse_work(self.case)
            self.R = self.case.h_q
        elif name == "sparse_prefill":
            self.case = W.sparse_prefill(seed=seed, device=dev)
            self.kind = "prefill"
            self.work = prefill_work(self.case)
            self.R = self.case.h_q
        elif name in ("sparse", "sparse_v41", "sparse_v41_fp4"):
            self.case = W.WORKLOADS[name](seed=seed, device=dev)
            self.kind = "sparse"
            self.work = sparse_work(self.case)
            self.R = self.case.h_q
        else:
            raise ValueError(name)
        c = self.case
        self.parts = B.mla_num_sm_parts(self.R, 1, dev)
        if self.kind == "prefill":
            self.out = torch.empty((c.s_q, c.h_q, c.d_v), dtype=torch.bfloat16, device=dev)
            self.lse = torch.empty((c.s_q, c.h_q), dtype=torch.float32, device=dev)
            self.ws = torch.empty((B.mla_sparse_prefill_workspace_size(c.s_q, c.h_q, c.topk,
                                                                       self.parts),),
                                  dtype=torch.uint8, device=dev)
            return
        b = c.batch
        if self.kind == "dense":
            self.out = torch.empty((b, c.s_q, c.h_q, c.d_v), dtype=torch.bfloat16, device=dev)
            self.lse = torch.empty((b, c.s_q, c.h_q), dtype=torch.float32, device=dev)
            self.ws = torch.empty((B.mla_workspace_size(b, self.R, c.d_v, self.parts),),
                                  dtype=torch.uint8, device=dev)
        elif self.kind in ("fused", "fused_sparse"):
            self.out = torch.empty((b, 1, c.h_q, 576), dtype=torch.uint8, device=dev)
            self.scale = torch.empty((b, 1, c.h_q), dtype=torch.float32, device=dev)
            self.lse = torch.empty((b, 1, c.h_q), dtype=torch.float32, device=dev)
            nbytes = (B.mla_fused_workspace_size(b, self.R, self.parts) if self.kind == "fused"
                      else B.mla_sparse_fused_workspace_size(b, c.h_q, c.topk, self.parts))
            self.ws = torch.empty((nbytes,), dtype=torch.uint8, device=dev)
        else:
            self.out = torch.empty((b, c.s_q, c.h_q, c.d_v), dtype=torch.bfloat16, device=dev)
            self.lse = torch.empty((b, c.s_q, c.h_q), dtype=torch.float32, device=dev)
            nbytes = (B.mla_sparse_workspace_size(b, c.s_q, c.h_q, c.topk, c.d_v, self.parts)
                      if name == "sparse" else
                      B.mla_sparse_v41_workspace_size(b, c.s_q, c.h_q, c.topk, self.parts))
            self.ws = torch.empty((nbytes,), dtype=torch.uint8, device=dev)
        if self.kind in ("dense", "fused"):
            self.meta = torch.empty((self.parts, 8), dtype=torch.int32, device=dev)
            self.ns = torch.empty((b + 1,), dtype=torch.int32, device=dev)

    def plan_summary(self):
        """The split plan of a step: partitions, splits and sequences split
        (from the host planner, bit-identical to the device planner the step
        runs), for the lengths the attention kernel sees."""
        c = self.case
        if self.kind in ("dense", "fused"):
            lengths = c.cache_seqlens.cpu()
        elif self.kind == "prefill":
            lengths = (c.topk_length.cpu() if c.topk_length is not None
                       else (c.indices.cpu() >= 0).sum(-1).to(torch.int32))
        else:
            lengths = (c.indices.cpu() >= 0).sum(-1).reshape(-1).to(torch.int32)
        lengths = lengths.to(torch.int32)
        parts = self.parts
        if self.kind == "prefill":
            lengths = lengths[:8192].clamp(0, c.topk)  # one launch
            parts = min(parts, self.B.mla_num_sms(self.dev) // (2 * -(-c.h_q // 128)))
        _, ns = self.B.mla_get_metadata_host(lengths, self.R, parts)
        per = (ns[1:] - ns[:-1]).tolist()
        return {"num_sm_parts": parts, "splits": int(ns[-1]),
                "sequences_split": int(sum(1 for n in per if n > 1)), "max_splits": int(max(per))}

    def attention_launches_per_step(self):
        return -(-self.case.s_q // 8192) if self.kind == "prefill" else 1

    def launches_per_step(self):
        # planner + attention kernel + combine (+ the FP8 gather for sparse, +
        # the query prologue for fused); the prefill runs lengths, planner,
        # attention and combine per launch of up to 8192 query tokens
        if self.kind == "prefill":
            c = self.case
            return 4 * -(-c.s_q // 8192)
        return 3 + (self.kind in ("sparse", "fused_sparse")) + (self.kind in ("fused", "fused_sparse"))

    def step(self, q=None):
        B, c = self.B, self.case
        if self.kind == "dense":
            m, n, _ = B.mla_get_metadata(c.cache_seqlens, self.R, 1, self.parts)
            B.mla_decode_fwd(c.q if q is None else q, c.kcache, c.block_table, c.cache_seqlens,
                             c.d_v, m, n, self.parts, causal=c.causal,
                             softmax_scale=c.softmax_scale, out=self.out, lse=self.lse,
                             workspace=self.ws)
        elif self.kind == "fused":
            m, n, _ = B.mla_get_metadata(c.cache_seqlens, self.R, 1, self.parts)
            B.mla_fused_norm_rope_attn_rope_cast(
                c.q_raw if q is None else q, c.gain, c.eps, c.rope_base, c.kcache,
                c.block_table, c.cache_seqlens, m, n, self.parts,
                softmax_scale=c.softmax_scale, out=self.out, out_scale=self.scale, lse=self.lse,
                workspace=self.ws)
        elif self.kind == "prefill":
            B.mla_sparse_prefill_fwd(c.q if q is None else q, c.kv, c.indices, c.softmax_scale,
                                     topk_length=c.topk_length, attn_sink=c.attn_sink,
                                     num_sm_parts=self.parts, out=self.out, lse=self.lse,
                                     workspace=self.ws)
        elif self.kind == "fused_sparse":
            B.mla_sparse_fused_norm_rope_attn_rope_cast(
                c.q_raw if q is None else q, c.gain, c.eps, c.rope_base, c.positions, c.kcache,
                c.indices, c.softmax_scale, self.parts, out=self.out, out_scale=self.scale,
                lse=self.lse, workspace=self.ws)
        else:
            B.mla_sparse_decode(c.q if q is None else q, c.kcache, c.indices, c.d_v,
                                c.softmax_scale, self.parts, out=self.out, lse=self.lse,
                                workspace=self.ws)

    def query(self):
        return self.case.q_raw if self.kind in ("fused", "fused_sparse") else self.case.q

    def with_own_buffers(self):
        """A second handle on the same inputs with its own outputs, workspace
        and scheduler buffers, so that several steps can be in flight at once."""
        import copy
        other = copy.copy(self)
        other.out = torch.empty_like(self.out)
        other.lse = torch.empty_like(self.lse)
        other.ws = torch.empty_like(self.ws)
        if hasattr(self, "scale"):
            other.scale = torch.empty_like(self.scale)
        if hasattr(self, "meta"):
            other.meta = torch.empty_like(self.meta)
            other.ns = torch.empty_like(self.ns)
        return other

    def outputs(self):
        return [self.out, self.lse] + ([self.scale] if self.kind in ("fused", "fused_sparse")
                                       else [])

    def capture(self):
        """One step recorded as a CUDA graph (planner, attention kernel,
        combine and, for sparse, the gather, with their programmatic launch
        edges).  Replays run the same launches on the same buffers without
        the host-side argument checks and launch calls of the API."""
        side = torch.cuda.Stream(self.dev)
        side.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(side):
            for _ in range(2):
                self.step()
        torch.cuda.current_stream(self.dev).wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.step()
        return g


class ClockSampler:
    """SM clock and throttle reasons of the bench's GPU sampled through NVML
    every ~2 ms on a background thread while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, dev):
        import threading
        self.samples = []
        self.h = None
        self.stop_flag = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(dev)
            try:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(dev.index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception:
            self.h = None
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self.stop_flag.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                self.samples.append((mhz, int(self.reasons_fn(self.h))))
            except Exception:
                return
            time.sleep(0.002)

    def start(self):
        if self.h is not None:
            self.thread.start()
        return self

    def stop(self):
        if self.h is None:
            return None
        self.stop_flag.set()
        self.thread.join(timeout=5)
        if not self.samples:
            return None
        reasons = set()
        for _, bits in self.samples:
            for bit, name in self.REASONS.items():
                if bits & bit:
                    reasons.add(name)
        mhz = [m for m, _ in self.samples]
        return {"sm_mhz": statistics.median(mhz), "sm_min_mhz": min(mhz),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(mhz), "source": "nvml"}


def sample_clocks_start(dev_index):
    """Fallback when NVML is unavailable: nvidia-smi sampling every 200 ms into
    a temporary CSV."""
    import tempfile
    path = os.path.join(tempfile.gettempdir(), f"mla_bench_clocks_{os.getpid()}.csv")
    try:
        f = open(path, "w")
        p = subprocess.Popen(
            ["nvidia-smi", f"--id={dev_index}",
             "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
             "--format=csv,noheader,nounits", "-lms", "200"], stdout=f, stderr=subprocess.DEVNULL)
        return p, f, path
    except Exception:
        return None, None, None


def sample_clocks_stop(handle):
    p, f, path = handle
    if p is None:
        return None
    p.terminate()
    try:
        p.wait(timeout=5)
    except Exception:
        p.kill()
    f.close()
    sm, mx, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in open(path):
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 8:
            continue
        try:
            sm.append(float(parts[0]))
            mx.append(float(parts[1]))
        except ValueError:
            continue
        for nm, v in zip(names, parts[4:8]):
            if v.lower() == "active":
                reasons.add(nm)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
            "samples": len(sm)}


def reduce_over_ranks(times, work, world, device):
    """Whole-job figures of a replicas-only run: every per-step time is the
    maximum over the ranks (the slowest replica ends the step) and the work is
    the sum over the ranks.  Every rank takes the same two collectives."""
    t = torch.tensor(times, dtype=torch.float64, device=device)
    w = torch.tensor(work, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        torch.distributed.all_reduce(w, op=torch.distributed.ReduceOp.SUM)
    return [float(x) for x in t], [float(x) for x in w]


def roofline_of(bound, flops, total_bytes, ms_kernel, peaks, peak_src, traffic=None):
    """Roofline entry of one attention launch of `ms_kernel` ms.  The launch is
    timed alone over a short run (well under a second), so a tensor-bound
    kernel is held against the burst bf16 peak; its HBM fraction is printed
    beside it (a kernel at the ridge needs both)."""
    s = ms_kernel * 1e-3
    gbs = total_bytes / s / 1e9
    if bound == "tensor":
        achieved = flops / s / 1e12
        peak = peaks["bf16_tflops"]
        return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} bf16 burst (kernel timed alone, short run)",
                "hbm_achieved_gbs": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
                "traffic": traffic, "kernel_ms": round(ms_kernel, 5)}
    peak = peaks["hbm_gbs"]
    return {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
            "frac": round(gbs / peak, 4), "peak_source": f"{peak_src} hbm copy",
            "traffic": traffic, "kernel_ms": round(ms_kernel, 5)}


def attention_kernel_ms(gs, steps, graph, dev):
    """Mean duration of the attention kernel over `steps` steps, between two
    CUDA events that the library records on its launching stream right before
    and right after that launch (mla_set_kernel_events).  With `graph`, the
    steps and their event records are captured as one CUDA graph and replayed
    once, so that the events do not include the host-side launch latency of a
    direct call; the events still sit between the step's launches, so no
    programmatic overlap with the planner or the combine enters the time."""
    st = torch.cuda.current_stream(dev)
    ks = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ke = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for e in ks + ke:
        e.record(st)  # creates the CUDA event behind the handle
    torch.cuda.synchronize(dev)
    if graph:
        g = torch.cuda.CUDAGraph()
        try:
            with torch.cuda.graph(g):
                for i in range(steps):
                    gs.B.mla_set_kernel_events(ks[i], ke[i])
                    gs.step()
        finally:
            gs.B.mla_set_kernel_events(None, None)
        g.replay()
        torch.cuda.synchronize(dev)
        del g
    else:
        for i in range(steps):
            gs.B.mla_set_kernel_events(ks[i], ke[i])
            gs.step()
        torch.cuda.synchronize(dev)
        gs.B.mla_set_kernel_events(None, None)
    return sum(a.elapsed_time(b) for a, b in zip(ks, ke)) / steps


def time_steps(gs, steps, graph, dev):
    """(ms per step, ms per attention launch) of `steps` steps: the steps as
    CUDA graph replays (or direct calls) with nothing between them, then the
    attention kernel alone in a second pass between library-recorded events."""
    st = torch.cuda.current_stream(dev)
    run = gs.step
    if graph:
        g = gs.capture()
        for _ in range(3):
            g.replay()
        run = g.replay
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(st)
    for _ in range(steps):
        run()
    ev1.record(st)
    torch.cuda.synchronize(dev)
    ms_step = ev0.elapsed_time(ev1) / steps
    return ms_step, attention_kernel_ms(gs, steps, graph, dev)


def measure_side(name, args, dev, peaks, peak_src):
    """The HBM-bound workloads measured in the same run as the headline one:
    step time, attention-kernel time, KV-read GB/s and the HBM roofline
    fraction of that kernel."""
    gs = GpuStep(name, seed=args.seed, dev=dev)
    for _ in range(max(3, args.warmup)):
        gs.step()
    torch.cuda.synchronize(dev)
    if gs.B.device_status() != 0:
        raise RuntimeError(f"device status set after warm-up of {name}")
    ms_step, ms_kernel = time_steps(gs, args.steps, args.graph, dev)
    flops, kv_bytes, total_bytes = gs.work
    roof = roofline_of(WORKLOAD_INFO[name][1], flops, total_bytes, ms_kernel, peaks, peak_src,
                       load_traffic(name))
    out = {"workload": WORKLOAD_INFO[name][0], "ms_per_step": round(ms_step, 5),
           "tflops": round(flops / (ms_step * 1e-3) / 1e12, 3),
           "kv_read_gbs": round(kv_bytes / (ms_step * 1e-3) / 1e9, 1),
           "kernel_ms": round(ms_kernel, 5), "roofline": roof}
    del gs
    torch.cuda.empty_cache()
    return out


E2E_IN_FLIGHT = 3  # end-to-end steps in flight (streams with their own buffers)


def run_gpu_arm(args, rank, world):
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    gs = GpuStep(args.workload, seed=args.seed + rank, dev=dev)
    flops, kv_bytes, total_bytes = gs.work
    st = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        gs.step()
    torch.cuda.synchronize(dev)
    status = gs.B.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status:#x} after warm-up")

    if world > 1:
        torch.distributed.barrier()
    sampler = ClockSampler(dev).start()
    clk = None if sampler.h is not None else sample_clocks_start(dev.index)
    torch.cuda.synchronize(dev)
    # the timed step: a CUDA graph replay of one API step (the direct calls
    # with --graph 0); a replay must reproduce the direct call's outputs
    run = gs.step
    if args.graph:
        gs.step()
        torch.cuda.synchronize(dev)
        ref = [t.clone() for t in gs.outputs()]
        graph = gs.capture()
        for t in gs.outputs():
            t.zero_()
        graph.replay()
        torch.cuda.synchronize(dev)
        if not all(torch.equal(a, b) for a, b in zip(ref, gs.outputs())):
            raise RuntimeError("CUDA graph replay differs from the direct call")
        for _ in range(3):
            graph.replay()
        run = graph.replay
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(st)
    for i in range(args.steps):
        run()
    ev1.record(st)
    torch.cuda.synchronize(dev)
    ms_total = ev0.elapsed_time(ev1)
    if world > 1:
        torch.distributed.barrier()
    # a second pass of the same K steps times the attention kernel alone: the
    # event records between launches would break the programmatic overlap of
    # consecutive launches, so they stay out of the step timing above
    torch.cuda.synchronize(dev)
    ms_kernel = attention_kernel_ms(gs, args.steps, args.graph, dev)
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if clk is None else sample_clocks_stop(clk)

    # end to end through the same API with host buffers: every step copies its
    # query in from pinned host memory, runs, and copies O and LSE back.  Three
    # steps are in flight on three streams, each with its own device buffers,
    # so that the host-to-device copies, the kernels and the device-to-host
    # copies of consecutive steps overlap as a serving loop runs them (with two,
    # a stream's next upload waits for its previous download and the copy
    # engine idles); the region ends when every stream has drained.
    ref_out = gs.out.cpu()
    q_dev = gs.query()
    q_host = q_dev.cpu().pin_memory()
    slots = [gs] + [gs.with_own_buffers() for _ in range(E2E_IN_FLIGHT - 1)]
    streams = [torch.cuda.Stream(dev) for _ in slots]
    q_bufs = [torch.empty_like(q_dev) for _ in slots]
    out_hosts = [torch.empty(gs.out.shape, dtype=gs.out.dtype).pin_memory() for _ in slots]
    lse_hosts = [torch.empty(gs.lse.shape, dtype=gs.lse.dtype).pin_memory() for _ in slots]
    has_scale = hasattr(gs, "scale")  # fused outputs: codes, scales and LSE
    scale_hosts = [torch.empty(gs.scale.shape, dtype=gs.scale.dtype).pin_memory()
                   for _ in slots] if has_scale else None

    def e2e_step(i):
        k = i % len(slots)
        with torch.cuda.stream(streams[k]):
            q_bufs[k].copy_(q_host, non_blocking=True)
            slots[k].step(q_bufs[k])
            out_hosts[k].copy_(slots[k].out, non_blocking=True)
            lse_hosts[k].copy_(slots[k].lse, non_blocking=True)
            if has_scale:
                scale_hosts[k].copy_(slots[k].scale, non_blocking=True)

    e2e_steps = max(4, min(args.steps, 50))
    torch.cuda.synchronize(dev)
    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for sk in streams:
        sk.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    for sk in streams:
        st.wait_stream(sk)
    e1.record(st)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if not all(torch.equal(h, ref_out) for h in out_hosts):
        raise RuntimeError("end-to-end outputs differ from the device-timed step's")
    status = gs.B.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status:#x} after timing")

    ms_step = ms_total / args.steps
    case_for_cpu = gs.case
    (ms_step, e2e_ms, ms_kernel), (flops_all, kv_all) = reduce_over_ranks(
        [ms_step, e2e_ms, ms_kernel], [flops, kv_bytes], world, dev)
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    desc, bound = WORKLOAD_INFO[args.workload]
    tflops = flops_all / (ms_step * 1e-3) / 1e12
    gbs = kv_all / (ms_step * 1e-3) / 1e9
    # dominant kernel: the attention kernel, timed alone; a workload with
    # several attention launches per step (the prefill's passes) is held to
    # the roofline over the whole step instead
    flops, _, total_bytes = gs.work
    multi = gs.attention_launches_per_step() > 1
    roof = roofline_of(bound, flops, total_bytes, ms_step if multi else ms_kernel, peaks, peak_src,
                       load_traffic(args.workload))
    if multi:
        roof["timed"] = (f"whole step ({gs.attention_launches_per_step()} attention launches "
                         "and their gathers, planners and combines)")
    line = {
        "metric": METRIC,
        "value": round(tflops, 3),
        "unit": "TFLOPS",
        "kv_read_gbs": round(gbs, 1),
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if ("sparse" not in args.workload or args.workload == "sparse_prefill") else
        "bf16 (fp4 cache dequantised)" if args.workload.endswith("fp4") else "bf16 (fp8 cache dequantised)",
        "data": "synthetic",
        "config": {"workload": desc, "name": args.workload,
                   "l2": "inputs larger than L2 (no flush)", "parallelism": f"replicas x{world}",
                   "launch": "CUDA graph replay of one API step" if args.graph
                   else "direct API calls",
                   "plan": gs.plan_summary()},
        "e2e": {"value": round(flops_all / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOPS",
                "h2d_bytes_per_step": int(q_dev.numel() * q_dev.element_size()),
                "d2h_bytes_per_step": int(gs.out.numel() * gs.out.element_size() +
                                          gs.lse.numel() * 4 +
                                          (gs.scale.numel() * 4 if hasattr(gs, "scale") else 0)),
                "ms_per_step": round(e2e_ms, 5), "steps_in_flight": E2E_IN_FLIGHT},
        "gpu_launches": gs.launches_per_step() * args.steps,
        "roofline": roof,
        "clocks": clocks,
    }
    if args.side and world == 1 and args.workload == "compute":
        # the memory-bound configurations of the same metric, timed in this run
        del gs, slots
        torch.cuda.empty_cache()
        line["hbm_bound"] = {n: measure_side(n, args, dev, peaks, peak_src)
                             for n in ("memory", "fused")}
    if args.cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(args.workload, seed=args.seed, budget_s=args.cpu_budget,
                                            case=case_for_cpu)
    return line


# ------------------------------------------------------ CPU oracle (baseline)

def oracle_rows_timed(name, case, rows):
    import oracle
    if name in ("compute", "memory", "tiny"):
        c = case
        t0 = time.perf_counter()
        oracle.dense_decode(c.q.cpu(), c.kcache_cpu, c.block_table.cpu(), c.cache_seqlens.cpu(),
                            c.d_v, c.softmax_scale, causal=c.causal, rows=rows)
        return time.perf_counter() - t0
    if name in ("fused", "fused_b1"):
        c = case
        t0 = time.perf_counter()
        oracle.fused_decode(c.q_raw.cpu(), c.gain.cpu(), c.eps, c.rope_base, c.kcache_cpu,
                            c.block_table.cpu(), c.cache_seqlens.cpu(), c.softmax_scale,
                            rows=rows)
        return time.perf_counter() - t0
    c = case
    t0 = time.perf_counter()
    if name == "sparse_prefill":
        oracle.sparse_prefill(c.q.cpu(), c.kv.cpu(), c.indices.cpu(), c.softmax_scale,
                              topk_length=None if c.topk_length is None else c.topk_length.cpu(),
                              attn_sink=None if c.attn_sink is None else c.attn_sink.cpu(),
                              rows=rows)
    elif name == "fused_sparse":
        oracle.fused_sparse_decode(c.q_raw.cpu(), c.gain.cpu(), c.eps, c.rope_base,
                                   c.positions.cpu(), c.kcache_cpu, c.indices.cpu(),
                                   c.softmax_scale, rows=rows)
    elif name.startswith("sparse_v41"):
        oracle.sparse_decode_v41(c.q.cpu(), c.kcache_cpu, c.indices.cpu(), c.softmax_scale,
                                 rows=rows)
    else:
        oracle.sparse_decode(c.q.cpu(), c.kcache_cpu, c.indices.cpu(), c.d_v, c.softmax_scale,
                             rows=rows)
    return time.perf_counter() - t0


def total_rows_of(case):
    """Query rows (token, head) of a workload's case."""
    if isinstance(case, W.PrefillCase):
        return case.s_q * case.h_q
    return case.batch * (case.s_q if hasattr(case, "s_q") else 1) * case.h_q


def row_flops(name, case, rows):
    """Algorithmic FLOPs of the sampled rows (same counting as the GPU arm)."""
    f = 0
    if name == "sparse_prefill":
        ix = case.indices.cpu()
        if case.topk_length is not None:
            n = case.topk_length.cpu().clamp(0, case.topk)
            ix = torch.where(torch.arange(case.topk)[None, :] < n[:, None], ix,
                             torch.full_like(ix, -1))
        valid = (ix >= 0).sum(-1).tolist()
        for r in rows:
            f += 2 * valid[r // case.h_q] * (576 + case.d_v)
        return f
    if name in ("compute", "memory", "tiny"):
        sl = case.cache_seqlens.cpu().tolist()
        for r in rows:
            b = r // (case.s_q * case.h_q)
            i = (r // case.h_q) % case.s_q
            L = sl[b]
            vis = max(0, min(L, L - case.s_q + 1 + i)) if case.causal else L
            f += 2 * vis * (576 + case.d_v)
    elif name in ("fused", "fused_b1"):
        sl = case.cache_seqlens.cpu().tolist()
        for r in rows:
            f += 2 * sl[r // case.h_q] * 1152
    else:
        valid = (case.indices.cpu() >= 0).sum(-1).reshape(-1).tolist()
        d_qk = sparse_dims(case)[0]
        for r in rows:
            f += 2 * valid[r // case.h_q] * (d_qk + case.d_v)
    return f


def make_case(name, seed, device="cpu"):
    """The named workload's seeded inputs."""
    if name in ("fused", "fused_b1"):
        return W.fused(seed=seed, device=device, batch=32 if name == "fused" else 1)
    return W.WORKLOADS[name](seed=seed, device=device)


def cpu_baseline(name, seed=0, budget_s=15.0, case=None):
    """Time the oracle as it stands on a bounded row sample of the workload."""
    import numpy as np
    import oracle
    if case is None:
        case = make_case(name, seed)
    if hasattr(case, "kcache"):
        case.kcache_cpu = case.kcache.cpu()
    total_rows = total_rows_of(case)
    rng = np.random.default_rng(seed)
    n = 8
    elapsed = oracle_rows_timed(name, case, np.sort(rng.choice(total_rows, n, replace=False)))
    per_row = max(elapsed / n, 1e-6)
    n = int(min(total_rows, max(8, budget_s / per_row)))
    rows = np.sort(rng.choice(total_rows, n, replace=False))
    elapsed = oracle_rows_timed(name, case, rows)
    f = row_flops(name, case, rows)
    return {"value": f / elapsed / 1e12, "unit": "TFLOPS", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": round(elapsed, 2),
            "sample": f"{n} of {total_rows} query rows (uniform random), fp64 C oracle, OpenMP"}


def run_reference_arm(args, rank, world):
    """The oracle timed on the host cores, each step a bounded row sample."""
    if rank != 0:
        return None
    desc, _ = WORKLOAD_INFO[args.workload]
    name = args.workload
    case = make_case(name, args.seed)
    per_step = max(1.0, args.cpu_budget / max(1, args.steps + args.warmup))
    import numpy as np
    import oracle
    if hasattr(case, "kcache"):
        case.kcache_cpu = case.kcache.cpu()
    total_rows = total_rows_of(case)
    rng = np.random.default_rng(args.seed)
    t8 = oracle_rows_timed(name, case, np.sort(rng.choice(total_rows, 8, replace=False))) / 8
    n = int(min(total_rows, max(4, per_step / max(t8, 1e-6))))
    times, fl = [], []
    for s in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(total_rows, n, replace=False))
        dt = oracle_rows_timed(name, case, rows)
        if s >= args.warmup:
            times.append(dt)
            fl.append(row_flops(name, case, rows))
    sec = sum(times)
    value = sum(fl) / sec / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec / len(times) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": desc, "name": name},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{n} of {total_rows} query rows per step, fp64 C oracle"},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="compute", choices=sorted(WORKLOAD_INFO))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--graph", type=int, default=1,
                    help="time CUDA graph replays of the step (0: direct API calls)")
    ap.add_argument("--side", type=int, default=1,
                    help="with the compute workload on one GPU, also time the memory and fused "
                         "(batch 32) workloads and print them under hbm_bound")
    ap.add_argument("--cpu-baseline", dest="cpu_baseline", type=int, default=1)
    ap.add_argument("--cpu-budget", dest="cpu_budget", type=float, default=15.0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            "nccl" if args.impl == "ours" else "gloo",
            timeout=datetime.timedelta(seconds=300))
    try:
        if args.impl == "reference":
            line = run_reference_arm(args, rank, world)
        else:
            line = run_gpu_arm(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
