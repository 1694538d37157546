"""Benchmark of the paged-KV attention library on one node.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Default workload: DECODE at the Llama-3-8B attention shape (batch 64, KV
lengths uniform in 512..8192, Hq 32, Hkv 8, D 128, bf16, page size 1 with
shuffled slots in a 600k-slot pool).  One step = one attn_plan followed by 32
layer calls of attn_decode_paged, each layer with its own pool (78.6 GB in
total, so every step reads inputs far larger than L2).  The metric is the
decode's algorithmic KV bandwidth: K and V rows read once, slot ids, Q and O,
divided by the device time.  Other workloads (``--workload``):
decode_long_llama3_70b, extend_prefix, sage_decode, sage_sparse_decode,
sage_extend_prefix, decode_fp8_llama3_8b, decode_tiny.

Prints ONE JSON line on rank 0.  Under torchrun each rank runs an independent
replica on its own GPU (no collective on the data path); the time is the max
over ranks and the value the sum of all ranks' bytes over that time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "paged decode KV GB/s (% HBM peak); paged extend TFLOP/s (% bf16 peak)"


# --------------------------------------------------------------------------- utilities

def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """Samples the GPU's SM clock, power and clock-event (throttle) reasons while running.

    NVML is polled every 10 ms on a background thread (the GPU found by its UUID, so a
    CUDA_VISIBLE_DEVICES remapping cannot point it at another board); without NVML,
    ``nvidia-smi -lms 200`` is the fallback.  `mark_start` / `mark_end` bracket the timed
    region and the summary keeps only the samples stamped inside it."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, cuda_index: int, period_s: float = 0.01):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []          # (time, sm_mhz, max_mhz, reasons set)
        self.t0 = self.t1 = None
        self.source = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def _poll_nvml(self, nv, h):
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.monotonic(), float(sm), float(mx),
                                     {n for n, b in self.REASONS if bits & b}))
            except Exception:
                pass
            time.sleep(self.period)

    def _poll_smi(self):
        for line in self._proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            self.samples.append((time.monotonic(), sm, mx,
                                 {n for (n, _), v in zip(self.REASONS, parts[5:9]) if v.lower() == "active"}))

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self._thread = threading.Thread(target=self._poll_nvml, args=(nv, h), daemon=True)
            self.source = "nvml 10 ms"
        except Exception:
            try:
                self._proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.cuda_index), "--query-gpu=" + self.FIELDS,
                     "--format=csv,noheader,nounits", "-lms", "200"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self._thread = threading.Thread(target=self._poll_smi, daemon=True)
                self.source = "nvidia-smi 200 ms"
            except Exception:
                self._thread = None
        if self._thread is not None:
            self._thread.start()
            deadline = time.monotonic() + 5.0
            while not self.samples and time.monotonic() < deadline:
                time.sleep(0.005)
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._proc is not None:
            # a region shorter than the 200 ms period: wait (up to 1 s) for one sample after its start
            deadline = time.monotonic() + 1.0
            while (self.t0 is not None and not any(x[0] >= self.t0 for x in list(self.samples))
                   and time.monotonic() < deadline):
                time.sleep(0.02)
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        samples = list(self.samples)
        where = "in_region"
        if self.t0 is not None and self.t1 is not None:
            inside = [x for x in samples if self.t0 <= x[0] <= self.t1]
            if not inside:
                inside, where = [x for x in samples if x[0] >= self.t0][:1], "post_region"
            samples = inside
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "source": self.source}
        reasons = set().union(*(x[3] for x in samples))
        return {"sm_mhz": statistics.median(x[1] for x in samples), "sm_max_mhz": samples[-1][2],
                "reasons": sorted(reasons), "samples": len(samples), "window": where, "source": self.source}


# The sources each workload's kernels are built from; profiles/traffic.json is keyed by their hash,
# so a recorded DRAM traffic figure is reported only for the exact kernels it was taken on.
KERNEL_SOURCES = {
    "decode_llama3_8b": ("decode.cu", "common.cuh"),
    "decode_long_llama3_70b": ("decode.cu", "common.cuh"),
    "decode_tiny": ("decode.cu", "common.cuh"),
    "decode_fp8_llama3_8b": ("decode_fp8.cu", "decode.cu", "common.cuh"),
    "extend_prefix": ("extend_duo.cu", "gather.cuh", "kernels.h", "common.cuh", "tma.cuh"),
    "extend_prefix_page1": ("extend_duo.cu", "gather.cuh", "kernels.h", "common.cuh", "tma.cuh"),
    "sage_decode": ("sage.cu", "common.cuh", "tma.cuh"),
    "sage_sparse_decode": ("sage.cu", "common.cuh", "tma.cuh"),
    "sage_extend_prefix": ("sage_extend.cu", "common.cuh", "tma.cuh"),
}


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "paged_kv_flashattention_split_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key: str, src_hash: str):
    """ncu DRAM bytes per launch recorded under profiles/ for this exact kernel source, else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(kernel_key)
        if rec and rec.get("source_hash") == src_hash:
            return float(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def init_ranks(world: int, local: int, backend: str):
    """One process per GPU under torchrun: join the process group (None when alone)."""
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    if backend == "nccl":
        torch.cuda.set_device(local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    return dist


def max_over_ranks(dist, value: float, device="cpu") -> float:
    """The job's time is the slowest rank's device time."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms_per_step: float, scale: float) -> float:
    """Whole-job throughput: every rank's units over the max-over-ranks step time."""
    return units_per_rank * world / (ms_per_step * 1e-3) / scale


# --------------------------------------------------------------------------- decode workload

class DecodeWorkload:
    """plan + L layer decode calls; layers rotate over `distinct_pools` pools."""

    def __init__(self, spec: wl.Spec, device: str):
        import paged_kv_flashattention_split_b200 as pa
        self.pa, self.spec, self.dev = pa, spec, device
        self.batch = wl.make_batch(spec, device)
        n_pools = spec.distinct_pools or spec.layers
        self.pools = [wl.make_bf16_pools(spec, self.batch, l, device) for l in range(n_pools)]
        self.q = [wl.make_bf16_queries(spec, spec.batch, l, device) for l in range(spec.layers)]
        self.out = [torch.empty_like(x) for x in self.q]
        self.params = pa.make_params(pa.PA_MODE_DECODE, spec.batch, spec.hq, spec.hkv, spec.head_dim,
                                     spec.page_size, max_kv_len=self.batch.page_table.shape[1] * spec.page_size)
        self.ws = torch.zeros(pa.pa_plan_workspace_size(self.params), dtype=torch.uint8, device=device)
        self.stream = torch.cuda.current_stream()
        L = self.batch.seq_lens.cpu().tolist()
        self.layer_bytes = wl.decode_kv_bytes(L, spec.hkv, spec.head_dim, 2, spec.page_size, spec.hq, 2, 2)
        self.step_bytes = self.layer_bytes * spec.layers
        self.launches_per_step = 1 + 2 * spec.layers

    def pool(self, l):
        return self.pools[l % len(self.pools)]

    def layer(self, l):
        k, v = self.pool(l)
        self.pa.attn_decode_paged(self.params, self.ws, self.q[l], k, v, self.batch.page_table,
                                  self.spec.sm_scale, self.out[l])

    def step(self):
        self.pa.attn_plan(self.params, self.batch.seq_lens, None, self.ws)
        for l in range(self.spec.layers):
            self.layer(l)

    # end to end: inputs from pinned host buffers, result read back, every step
    def setup_e2e(self):
        self.h_q = [x.cpu().pin_memory() for x in self.q]
        self.h_lens = self.batch.seq_lens.cpu().pin_memory()
        self.h_table = self.batch.page_table.cpu().pin_memory()
        self.h_out = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in self.out]
        self.e2e_h2d = sum(x.numel() * 2 for x in self.h_q) + self.h_lens.numel() * 4 + self.h_table.numel() * 4
        self.e2e_d2h = sum(x.numel() * 2 for x in self.h_out)

    def step_e2e(self):
        self.batch.seq_lens.copy_(self.h_lens, non_blocking=True)
        self.batch.page_table.copy_(self.h_table, non_blocking=True)
        self.pa.attn_plan(self.params, self.batch.seq_lens, None, self.ws)
        for l in range(self.spec.layers):
            self.q[l].copy_(self.h_q[l], non_blocking=True)
            self.layer(l)
            self.h_out[l].copy_(self.out[l], non_blocking=True)

    # the oracle on a bounded sample of the same workload (host cores)
    def oracle_sample(self, seconds=12.0):
        from oracle import attention as oa
        spec = self.spec
        t0 = time.perf_counter()
        table = self.batch.page_table.cpu().numpy()
        lens = self.batch.seq_lens.cpu().numpy()
        k, v = self.pool(0)
        kb = k.view(torch.int16).cpu().numpy().view(np.uint16)
        vb = v.view(torch.int16).cpu().numpy().view(np.uint16)
        qb = self.q[0].view(torch.int16).cpu().numpy().view(np.uint16)
        prep = time.perf_counter() - t0
        done, nbytes, r = 0.0, 0.0, 0
        t0 = time.perf_counter()
        while r < spec.batch and (time.perf_counter() - t0) < seconds:
            oa.decode(qb[r:r + 1], kb, vb, table[r:r + 1], lens[r:r + 1], spec.page_size, spec.sm_scale)
            nbytes += wl.decode_kv_bytes([int(lens[r])], spec.hkv, spec.head_dim, 2, spec.page_size, spec.hq, 2, 2)
            r += 1
        done = time.perf_counter() - t0
        return nbytes, done, f"oracle.attention.decode on requests 0..{r - 1} of layer 0 ({r} of {spec.batch} requests, {int(lens[:r].sum())} keys); host copy {prep:.1f}s untimed"


class SageWorkload(DecodeWorkload):
    """plan + L layer calls of the 8-bit Sage decode, each layer with its own 8-bit pools."""

    def __init__(self, spec: wl.Spec, device: str):
        import paged_kv_flashattention_split_b200 as pa
        self.pa, self.spec, self.dev = pa, spec, device
        self.batch = wl.make_batch(spec, device)
        n_pools = spec.distinct_pools or spec.layers
        self.layers_data = [wl.make_sage_layer(spec, self.batch, l, device) for l in range(n_pools)]
        self.q = [self.layers_data[l % n_pools].q8 for l in range(spec.layers)]
        self.out = [torch.empty((spec.batch, spec.hq, spec.head_dim), dtype=torch.bfloat16, device=device)
                    for _ in range(spec.layers)]
        self.params = pa.make_params(pa.PA_MODE_SAGE_DECODE, spec.batch, spec.hq, spec.hkv, spec.head_dim, 64,
                                     max_kv_len=self.batch.page_table.shape[1] * 64, sage_k_block=64)
        self.ws = torch.zeros(pa.pa_plan_workspace_size(self.params), dtype=torch.uint8, device=device)
        L = self.batch.seq_lens.cpu().tolist()
        # K8 + V8 rows (1 B each), one sfK per 64-key block and head, page ids, Q8 + sfQ, bf16 O
        self.layer_bytes = float(sum(L) * spec.hkv * spec.head_dim * 2
                                 + sum((x + 63) // 64 for x in L) * (spec.hkv * 4 + 4)
                                 + spec.batch * spec.hq * (spec.head_dim * 1 + 4 + spec.head_dim * 2))
        self.step_bytes = self.layer_bytes * spec.layers
        self.launches_per_step = 1 + 3 * spec.layers   # plan, then score + value + merge per layer

    def layer(self, l):
        d = self.layers_data[l % len(self.layers_data)]
        self.pa.attn_decode_paged_sage(self.params, self.ws, d.q8, d.sf_q, d.k8, d.v8, d.sf_k, d.sf_v, d.v_mean,
                                       self.batch.page_table, self.out[l])

    def setup_e2e(self):
        self.h_q = [x.cpu().pin_memory() for x in self.q]
        self.h_lens = self.batch.seq_lens.cpu().pin_memory()
        self.h_table = self.batch.page_table.cpu().pin_memory()
        self.h_out = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in self.out]
        self.e2e_h2d = sum(x.numel() for x in self.h_q) + self.h_lens.numel() * 4 + self.h_table.numel() * 4
        self.e2e_d2h = sum(x.numel() * 2 for x in self.h_out)

    def oracle_sample(self, seconds=12.0):
        from oracle import sage as osg
        spec = self.spec
        d = self.layers_data[0]
        host = {k: getattr(d, k).cpu().numpy() for k in ("q8", "sf_q", "k8", "v8", "sf_k", "sf_v", "v_mean")}
        table = self.batch.page_table.cpu().numpy()
        lens = self.batch.seq_lens.cpu().numpy()
        nbytes, r = 0.0, 0
        t0 = time.perf_counter()
        while r < spec.batch and (time.perf_counter() - t0) < seconds:
            osg.sage_decode(host["q8"][r:r + 1], host["sf_q"][r:r + 1], host["k8"], host["v8"], host["sf_k"],
                            host["sf_v"], host["v_mean"], table[r:r + 1], lens[r:r + 1], 64)
            nbytes += self.layer_bytes * float(lens[r]) / float(lens.sum())
            r += 1
        return nbytes, time.perf_counter() - t0, f"oracle.sage.sage_decode on requests 0..{r - 1} of layer 0"


class ExtendWorkload(DecodeWorkload):
    """plan + L layer calls of the causal paged extend, each layer with its own pools."""

    def __init__(self, spec: wl.Spec, device: str):
        import paged_kv_flashattention_split_b200 as pa
        self.pa, self.spec, self.dev = pa, spec, device
        self.batch = wl.make_batch(spec, device)
        n_pools = spec.distinct_pools or spec.layers
        self.pools = [wl.make_bf16_pools(spec, self.batch, l, device) for l in range(n_pools)]
        self.total_q = int(self.batch.cu_seqlens_q[-1])
        self.q = [wl.make_bf16_queries(spec, self.total_q, l, device) for l in range(spec.layers)]
        self.out = [torch.empty_like(x) for x in self.q]
        self.params = pa.make_params(pa.PA_MODE_EXTEND, spec.batch, spec.hq, spec.hkv, spec.head_dim,
                                     spec.page_size, max_kv_len=self.batch.page_table.shape[1] * spec.page_size,
                                     max_q_tokens=self.total_q)
        self.ws = torch.zeros(pa.pa_plan_workspace_size(self.params), dtype=torch.uint8, device=device)
        L = self.batch.seq_lens.cpu().tolist()
        n = self.batch.new_lens.cpu().tolist()
        pairs = sum(ni * (Li - ni) + ni * (ni + 1) // 2 for Li, ni in zip(L, n))   # unmasked (q, k) pairs
        self.layer_flops = 4.0 * spec.head_dim * spec.hq * pairs
        self.step_flops = self.layer_flops * spec.layers
        self.layer_bytes = self.layer_flops          # the metric for this workload is TFLOP/s
        self.step_bytes = self.step_flops
        self.unit, self.scale = "TFLOP/s", 1e12
        self.launches_per_step = 1 + spec.layers

    def layer(self, l):
        k, v = self.pool(l)
        self.pa.attn_extend_paged(self.params, self.ws, self.q[l], k, v, self.batch.page_table,
                                  self.spec.sm_scale, self.out[l])

    def step_e2e(self):
        self.batch.seq_lens.copy_(self.h_lens, non_blocking=True)
        self.batch.cu_seqlens_q.copy_(self.h_cu, non_blocking=True)
        self.batch.page_table.copy_(self.h_table, non_blocking=True)
        self.pa.attn_plan(self.params, self.batch.seq_lens, self.batch.cu_seqlens_q, self.ws)
        for l in range(self.spec.layers):
            self.q[l].copy_(self.h_q[l], non_blocking=True)
            self.layer(l)
            self.h_out[l].copy_(self.out[l], non_blocking=True)

    def step(self):
        self.pa.attn_plan(self.params, self.batch.seq_lens, self.batch.cu_seqlens_q, self.ws)
        for l in range(self.spec.layers):
            self.layer(l)

    def setup_e2e(self):
        super().setup_e2e()
        self.h_cu = self.batch.cu_seqlens_q.cpu().pin_memory()
        self.e2e_h2d += self.h_cu.numel() * 4

    def oracle_sample(self, seconds=12.0):
        from oracle import attention as oa
        spec = self.spec
        k, v = self.pool(0)
        kb = k.view(torch.int16).cpu().numpy().view(np.uint16)
        vb = v.view(torch.int16).cpu().numpy().view(np.uint16)
        qb = self.q[0].view(torch.int16).cpu().numpy().view(np.uint16)
        cu = self.batch.cu_seqlens_q.cpu().numpy()
        table = self.batch.page_table.cpu().numpy()
        lens = self.batch.seq_lens.cpu().numpy()
        flops, r, h = 0.0, 0, 0
        G = spec.hq // spec.hkv
        t0 = time.perf_counter()
        while (time.perf_counter() - t0) < seconds and r < spec.batch:
            q0, q1 = int(cu[r]), int(cu[r + 1])
            sub_cu = np.array([0, q1 - q0])
            oa.extend(qb[q0:q1, h:h + 1], sub_cu, kb[:, h // G:h // G + 1], vb[:, h // G:h // G + 1],
                      table[r:r + 1], lens[r:r + 1], spec.page_size, spec.sm_scale)
            n = q1 - q0
            flops += 4.0 * spec.head_dim * (n * (int(lens[r]) - n) + n * (n + 1) // 2)
            h += 1
            if h == spec.hq:
                h, r = 0, r + 1
        return flops, time.perf_counter() - t0, f"oracle.attention.extend, one query head at a time, {r * spec.hq + h} (request, head) pairs of layer 0"


class SageExtendWorkload(ExtendWorkload):
    """plan + L layer calls of the 8-bit Sage extend (page size 64), each layer with its own pools."""

    def __init__(self, spec: wl.Spec, device: str):
        import paged_kv_flashattention_split_b200 as pa
        self.pa, self.spec, self.dev = pa, spec, device
        self.batch = wl.make_batch(spec, device)
        self.total_q = int(self.batch.cu_seqlens_q[-1])
        n_pools = spec.distinct_pools or spec.layers
        self.layers_data = [wl.make_sage_layer(spec, self.batch, l, device, q_rows=self.total_q) for l in range(n_pools)]
        self.q = [self.layers_data[l % n_pools].q8 for l in range(spec.layers)]
        self.out = [torch.empty((self.total_q, spec.hq, spec.head_dim), dtype=torch.bfloat16, device=device)
                    for _ in range(spec.layers)]
        self.params = pa.make_params(pa.PA_MODE_EXTEND, spec.batch, spec.hq, spec.hkv, spec.head_dim, 64,
                                     max_kv_len=self.batch.page_table.shape[1] * 64, max_q_tokens=self.total_q)
        self.ws = torch.zeros(pa.pa_plan_workspace_size(self.params), dtype=torch.uint8, device=device)
        L = self.batch.seq_lens.cpu().tolist()
        n = self.batch.new_lens.cpu().tolist()
        pairs = sum(ni * (Li - ni) + ni * (ni + 1) // 2 for Li, ni in zip(L, n))   # unmasked (q, k) pairs
        # QK and PV over the unmasked pairs (the row-max pass is this design's own extra work)
        self.layer_flops = 4.0 * spec.head_dim * spec.hq * pairs
        self.step_flops = self.layer_flops * spec.layers
        self.layer_bytes = self.layer_flops
        self.step_bytes = self.step_flops
        self.unit, self.scale = "TFLOP/s", 1e12
        self.launches_per_step = 1 + spec.layers

    def layer(self, l):
        d = self.layers_data[l % len(self.layers_data)]
        self.pa.attn_extend_paged_sage(self.params, self.ws, d.q8, d.sf_q, d.k8, d.v8, d.sf_k, d.sf_v, d.v_mean,
                                       self.batch.page_table, self.out[l])

    def setup_e2e(self):
        self.h_q = [x.cpu().pin_memory() for x in self.q]
        self.h_lens = self.batch.seq_lens.cpu().pin_memory()
        self.h_table = self.batch.page_table.cpu().pin_memory()
        self.h_cu = self.batch.cu_seqlens_q.cpu().pin_memory()
        self.h_out = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in self.out]
        self.e2e_h2d = (sum(x.numel() for x in self.h_q) + self.h_lens.numel() * 4 + self.h_table.numel() * 4
                        + self.h_cu.numel() * 4)
        self.e2e_d2h = sum(x.numel() * 2 for x in self.h_out)

    def oracle_sample(self, seconds=12.0):
        from oracle import sage as osg
        spec = self.spec
        d = self.layers_data[0]
        host = {k: getattr(d, k).cpu().numpy() for k in ("q8", "sf_q", "k8", "v8", "sf_k", "sf_v", "v_mean")}
        cu = self.batch.cu_seqlens_q.cpu().numpy()
        table = self.batch.page_table.cpu().numpy()
        lens = self.batch.seq_lens.cpu().numpy()
        G = spec.hq // spec.hkv
        flops, r, h = 0.0, 0, 0
        t0 = time.perf_counter()
        while (time.perf_counter() - t0) < seconds and r < spec.batch:
            q0, q1 = int(cu[r]), int(cu[r + 1])
            hk = h // G
            osg.sage_extend(host["q8"][q0:q1, h:h + 1], host["sf_q"][q0:q1, h:h + 1], np.array([0, q1 - q0]),
                            host["k8"][:, hk:hk + 1], host["v8"][:, hk:hk + 1], host["sf_k"][:, hk:hk + 1],
                            host["sf_v"][hk:hk + 1], host["v_mean"][hk:hk + 1], table[r:r + 1], lens[r:r + 1], 64)
            nn = q1 - q0
            flops += 4.0 * spec.head_dim * (nn * (int(lens[r]) - nn) + nn * (nn + 1) // 2)
            h += 1
            if h == spec.hq:
                h, r = 0, r + 1
        return flops, time.perf_counter() - t0, f"oracle.sage.sage_extend, one query head at a time, {r * spec.hq + h} (request, head) pairs of layer 0"


class SageSparseWorkload(SageWorkload):
    """plan (with the batch's block mask) + L layer calls of the block-sparse Sage decode."""

    def __init__(self, spec: wl.Spec, device: str):
        super().__init__(spec, device)
        import paged_kv_flashattention_split_b200 as pa
        self.mask = wl.make_block_mask(spec, self.batch, device)
        self.params = pa.make_params(pa.PA_MODE_SAGE_SPARSE, spec.batch, spec.hq, spec.hkv, spec.head_dim, 64,
                                     max_kv_len=self.batch.page_table.shape[1] * 64, sage_k_block=64)
        self.ws = torch.zeros(pa.pa_plan_workspace_size(self.params), dtype=torch.uint8, device=device)
        L = self.batch.seq_lens.cpu().tolist()
        m = self.mask.cpu().numpy()
        sel = [sum(min(64, x - 64 * b) for b in range(-(-x // 64)) if m[r][b]) for r, x in enumerate(L)]
        nsel_blocks = sum(int(m[r][: -(-x // 64)].sum()) for r, x in enumerate(L))
        # the selected keys' K8 + V8 rows, their blocks' sfK and page ids, Q8 + sfQ, bf16 O
        self.layer_bytes = float(sum(sel) * spec.hkv * spec.head_dim * 2 + nsel_blocks * (spec.hkv * 4 + 4)
                                 + spec.batch * spec.hq * (spec.head_dim * 1 + 4 + spec.head_dim * 2))
        self.step_bytes = self.layer_bytes * spec.layers
        self.selected_keys = sum(sel)

    def step(self):
        self.pa.attn_plan_sage_sparse(self.params, self.batch.seq_lens, self.mask, self.ws)
        for l in range(self.spec.layers):
            self.layer(l)

    def step_e2e(self):
        self.batch.seq_lens.copy_(self.h_lens, non_blocking=True)
        self.batch.page_table.copy_(self.h_table, non_blocking=True)
        self.pa.attn_plan_sage_sparse(self.params, self.batch.seq_lens, self.mask, self.ws)
        for l in range(self.spec.layers):
            self.q[l].copy_(self.h_q[l], non_blocking=True)
            self.layer(l)
            self.h_out[l].copy_(self.out[l], non_blocking=True)

    def oracle_sample(self, seconds=12.0):
        from oracle import sage as osg
        spec = self.spec
        d = self.layers_data[0]
        host = {k: getattr(d, k).cpu().numpy() for k in ("q8", "sf_q", "k8", "v8", "sf_k", "sf_v", "v_mean")}
        table = self.batch.page_table.cpu().numpy()
        lens = self.batch.seq_lens.cpu().numpy()
        m = self.mask.cpu().numpy()
        t0 = time.perf_counter()
        nbytes, r = 0.0, 0
        while r < spec.batch and (time.perf_counter() - t0) < seconds:
            osg.sage_decode(host["q8"][r:r + 1], host["sf_q"][r:r + 1], host["k8"], host["v8"], host["sf_k"],
                            host["sf_v"], host["v_mean"], table[r:r + 1], lens[r:r + 1], 64, block_mask=m[r:r + 1])
            L = int(lens[r])
            nbytes += sum(min(64, L - 64 * b) for b in range(-(-L // 64)) if m[r][b]) * spec.hkv * spec.head_dim * 2
            r += 1
        return nbytes, time.perf_counter() - t0, f"oracle.sage.sage_decode (block mask) on requests 0..{r - 1} of layer 0"


class Fp8DecodeWorkload(DecodeWorkload):
    """plan + L layer calls of the FP8-KV decode (E4M3 pools, bf16 Q and O)."""

    def __init__(self, spec: wl.Spec, device: str):
        import paged_kv_flashattention_split_b200 as pa
        self.pa, self.spec, self.dev = pa, spec, device
        self.batch = wl.make_batch(spec, device)
        n_pools = spec.distinct_pools or spec.layers
        self.pools = [wl.make_fp8_pools(spec, self.batch, l, device) for l in range(n_pools)]
        self.q = [wl.make_bf16_queries(spec, spec.batch, l, device) for l in range(spec.layers)]
        self.out = [torch.empty_like(x) for x in self.q]
        self.params = pa.make_params(pa.PA_MODE_DECODE, spec.batch, spec.hq, spec.hkv, spec.head_dim,
                                     spec.page_size, max_kv_len=self.batch.page_table.shape[1] * spec.page_size)
        self.ws = torch.zeros(pa.pa_plan_workspace_size(self.params), dtype=torch.uint8, device=device)
        self.stream = torch.cuda.current_stream()
        L = self.batch.seq_lens.cpu().tolist()
        # K8 + V8 rows (1 B per element), page ids, bf16 Q and O
        self.layer_bytes = wl.decode_kv_bytes(L, spec.hkv, spec.head_dim, 1, spec.page_size, spec.hq, 2, 2)
        self.step_bytes = self.layer_bytes * spec.layers
        self.launches_per_step = 1 + 2 * spec.layers

    def layer(self, l):
        k8, v8 = self.pool(l)
        self.pa.attn_decode_paged_fp8(self.params, self.ws, self.q[l], k8, v8, wl.FP8_SCALE, wl.FP8_SCALE,
                                      self.batch.page_table, self.spec.sm_scale, self.out[l])

    def oracle_sample(self, seconds=12.0):
        from oracle import attention as oa
        spec = self.spec
        t0 = time.perf_counter()
        table = self.batch.page_table.cpu().numpy()
        lens = self.batch.seq_lens.cpu().numpy()
        k8, v8 = (x.cpu().numpy() for x in self.pool(0))
        qb = self.q[0].view(torch.int16).cpu().numpy().view(np.uint16)
        prep = time.perf_counter() - t0
        nbytes, r = 0.0, 0
        t0 = time.perf_counter()
        while r < spec.batch and (time.perf_counter() - t0) < seconds:
            oa.decode_fp8(qb[r:r + 1], k8, v8, wl.FP8_SCALE, wl.FP8_SCALE, table[r:r + 1], lens[r:r + 1],
                          spec.page_size, spec.sm_scale)
            nbytes += wl.decode_kv_bytes([int(lens[r])], spec.hkv, spec.head_dim, 1, spec.page_size, spec.hq, 2, 2)
            r += 1
        return nbytes, time.perf_counter() - t0, f"oracle.attention.decode_fp8 on requests 0..{r - 1} of layer 0 ({r} of {spec.batch} requests, {int(lens[:r].sum())} keys); host copy {prep:.1f}s untimed"


WORKLOADS = {   # workload name (workloads.SPECS) -> the step it runs
    "extend_prefix": ExtendWorkload,
    "extend_prefix_page1": ExtendWorkload,
    "decode_fp8_llama3_8b": Fp8DecodeWorkload,
    "sage_sparse_decode": SageSparseWorkload,
    "sage_extend_prefix": SageExtendWorkload,
    "sage_decode": SageWorkload,
    "decode_llama3_8b": DecodeWorkload,
    "decode_long_llama3_70b": DecodeWorkload,
    "decode_tiny": DecodeWorkload,
}


# --------------------------------------------------------------------------- main

DTYPES = {"sage_decode": "int8/e4m3 in, fp32 math, bf16 out",
          "sage_sparse_decode": "int8/e4m3 in, fp32 math, bf16 out",
          "sage_extend_prefix": "int8 x int8 -> int32 (QK) and e4m3 x e4m3 -> fp32 (PV) tensor-core math, bf16 out",
          "decode_fp8_llama3_8b": "e4m3 KV, bf16 Q/O, f16 tensor-core math, fp32 accumulation"}
STEP_CALLS = {"sage_decode": "attn_decode_paged_sage", "sage_sparse_decode": "attn_decode_paged_sage (block-sparse plan)",
              "sage_extend_prefix": "attn_extend_paged_sage", "extend_prefix": "attn_extend_paged",
              "extend_prefix_page1": "attn_extend_paged",
              "decode_fp8_llama3_8b": "attn_decode_paged_fp8"}
ROOFLINE_KERNELS = {
    "sage_decode": "attn_decode_paged_sage call (sage_score_kernel + sage_value_kernel + sage_merge_kernel)",
    "sage_sparse_decode": "attn_decode_paged_sage call, block-sparse plan (score + value + merge kernels)",
    "sage_extend_prefix": "sage_extend_kernel (one launch per attn_extend_paged_sage call; 3 contractions per tile pair, 2 counted)",
    "extend_prefix": "extend_duo_kernel (a pair of CTAs per query tile and 4 heads; one launch per attn_extend_paged call)",
    "extend_prefix_page1": "extend_duo_kernel with slot-by-slot cp.async gathers (page size 1; one launch per call)",
    "decode_fp8_llama3_8b": "attn_decode_paged_fp8 call (decode_fp8_kernel + merge_kernel)"}
# workloads measured beside the default decode in the default run (the other halves of the metric)
DEFAULT_EXTRAS = ("extend_prefix", "sage_decode")


def workload_config(name, spec, num_slots, world):
    """The `config` object of a JSON line: the workload itself, the same for both arms."""
    cfg = {
        "workload": name,
        "batch": spec.batch, "seq_lens": f"U[{spec.len_lo},{spec.len_hi}]", "hq": spec.hq, "hkv": spec.hkv,
        "head_dim": spec.head_dim, "page_size": spec.page_size, "layers": spec.layers,
        "distinct_pools": spec.distinct_pools or spec.layers, "pool_slots": num_slots,
        "step": "attn_plan + %d x %s" % (spec.layers, STEP_CALLS.get(name, "attn_decode_paged")),
        "l2": "inputs larger than L2 (the step's layers read their own pools, far more than L2)",
        "parallelism": f"replicas x{world}",
    }
    if spec.mode == "extend":
        cfg["new_lens"] = f"U[{spec.new_lo},{spec.new_hi}]"
    return cfg


def measure(name, spec, args, dist, world, local, rank, peaks, cpu_baseline=True):
    """Run one workload: warm-up, the timed steps (CUDA events, max over ranks), the CUDA-graph replay,
    the end-to-end run through host buffers, and (rank 0, one GPU) the oracle on a bounded sample.
    Returns the JSON fields of that workload."""
    hbm_peak, bf16_peak, bf16_sus, peak_src = peaks
    cls = WORKLOADS[name]
    dev = f"cuda:{local}"
    work = cls(spec, dev)
    torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        work.step()
    torch.cuda.synchronize()

    # timed region: CUDA events on the launching stream around the steps only.  No event sits
    # between two layer calls: an event recorded there would end each programmatic dependent
    # launch chain (the next call's first kernel could no longer start while the previous
    # call's last one drains), so the per-call figure below is the step time / layers.
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        clocks.mark_start()
        start.record()
        for _ in range(args.steps):
            work.step()
        end.record()
        torch.cuda.synchronize()
        clocks.mark_end()
    total_ms = max_over_ranks(dist, start.elapsed_time(end), dev)
    if dist is not None:
        dist.barrier()
    ms_per_step = total_ms / args.steps
    scale = getattr(work, "scale", 1e9)
    value = job_throughput(work.step_bytes, world, ms_per_step, scale)

    # the same step captured once in a CUDA graph and replayed (launch overhead removed)
    try:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                work.step()
        torch.cuda.synchronize()
        for _ in range(3):
            graph.replay()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        g0.record()
        for _ in range(args.steps):
            graph.replay()
        g1.record()
        torch.cuda.synchronize()
        g_ms = max_over_ranks(dist, g0.elapsed_time(g1) / args.steps, dev)
        graph_info = {"ms_per_step": round(g_ms, 4), "value": round(job_throughput(work.step_bytes, world, g_ms, scale), 1)}
        del graph
    except Exception as exc:  # reported, never silently replaced
        graph_info = {"error": str(exc)[:200]}

    # end to end through the public API with host buffers
    work.setup_e2e()
    for _ in range(2):
        work.step_e2e()
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(1, min(args.steps, 5))
    e_start.record()
    for _ in range(e_steps):
        work.step_e2e()
    e_end.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(dist, e_start.elapsed_time(e_end) / e_steps, dev)
    e2e_value = job_throughput(work.step_bytes, world, e2e_ms, scale)

    avg_layer_ms = ms_per_step / spec.layers   # one layer call, the once-per-step plan's share included
    achieved = work.layer_bytes / (avg_layer_ms * 1e-3) / scale
    kernel_src = KERNEL_SOURCES.get(name, KERNEL_SOURCES["decode_llama3_8b"])
    traffic = recorded_traffic(name, source_hash(*kernel_src))
    unit = getattr(work, "unit", "GB/s")
    clock_summary = clocks.summary()
    sustained = None
    if unit == "TFLOP/s":
        # tensor-bound: the burst bf16 figure (a kernel timed alone), and beside it the sustained
        # one (a kernel timed inside a long, power-capped step); the 8-bit contractions of the
        # Sage extend take 2x either (the nominal 8-bit : bf16 ratio)
        mult = 2.0 if name == "sage_extend_prefix" else 1.0
        what = "bf16 dense x 2 (8-bit dense = 2x bf16 nominal)" if mult == 2.0 else "bf16 dense"
        bound, peak = "tensor", round(mult * bf16_peak, 1)
        peak_note = (f"{peak_src} burst {what}; timed region {total_ms / 1000:.2f} s, SM clock median "
                     f"{clock_summary.get('sm_mhz')} MHz, reasons {clock_summary.get('reasons')}")
        sustained = {"peak": round(mult * bf16_sus, 1), "frac": round(achieved / (mult * bf16_sus), 4),
                     "note": f"{peak_src} sustained {what} (seconds-long loop under the power cap)"}
    else:
        bound, peak, peak_note = "hbm", hbm_peak, peak_src

    out = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": unit,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPES.get(name, "bf16"),
        "data": "synthetic",
        "config": workload_config(name, spec, work.batch.num_slots, world),
        "roofline": {
            "bound": bound, "achieved": round(achieved, 1), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "kernel": ROOFLINE_KERNELS.get(name, "attn_decode_paged call (decode_splitkv_kernel + merge_kernel)")
                      + ", per layer call: the timed region's CUDA-event time / (steps x layers), the once-per-step plan included",
            "peak_source": peak_note,
        },
        "e2e": {"value": round(e2e_value, 1), "unit": unit, "h2d_bytes_per_step": int(work.e2e_h2d),
                "d2h_bytes_per_step": int(work.e2e_d2h), "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": work.launches_per_step * args.steps,
        "graph": graph_info,
        "clocks": clock_summary,
    }
    if sustained is not None:
        out["roofline"]["sustained"] = sustained
    if cpu_baseline and rank == 0 and world == 1:
        nbytes, secs, sample = work.oracle_sample()
        out["cpu_baseline"] = {"value": round(nbytes / secs / scale, 6), "unit": unit, "cores": blas_threads(),
                               "kind": "oracle", "sample": sample}
    del work
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_llama3_8b", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="default workload only: skip the extend and Sage decode objects")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling only: fewer layer calls per step than the workload defines")
    ap.add_argument("--distinct-pools", type=int, default=0,
                    help="profiling only: allocate fewer pools (layers rotate over them)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = init_ranks(world, local, "gloo" if args.impl == "reference" else "nccl")

    def spec_for(name):
        spec = wl.SPECS[name]
        if args.layers:
            spec = spec.scaled(layers=args.layers)
        if args.distinct_pools:
            spec = spec.scaled(distinct_pools=args.distinct_pools)
        return spec

    spec = spec_for(args.workload)
    peaks = load_peaks()

    if args.impl == "reference":
        if rank != 0:
            if dist is not None:
                dist.destroy_process_group()
            return
        run_reference(args, spec, WORKLOADS[args.workload])
        if dist is not None:
            dist.destroy_process_group()
        return

    torch.cuda.set_device(f"cuda:{local}")
    line = measure(args.workload, spec, args, dist, world, local, rank, peaks, not args.no_cpu_baseline)
    # the default run also measures the extend half of the metric and the 8-bit Sage decode, each
    # in its own timed region with its own clocks (the decode's pools are freed first)
    if args.workload == "decode_llama3_8b" and not args.no_extras:
        for name in DEFAULT_EXTRAS:
            key = "extend" if name == "extend_prefix" else name
            line[key] = measure(name, spec_for(name), args, dist, world, local, rank, peaks,
                                not args.no_cpu_baseline)
            for k in ("metric", "n_gpus", "steps", "warmup", "higher_is_better", "scaling", "vs_baseline", "data"):
                line[key].pop(k, None)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args, spec, cls):
    """The oracle as it stands, on the host cores, on a bounded sample of the workload per step."""
    from oracle import attention as oa
    from oracle import sage as osg
    batch = wl.make_batch(spec, "cpu")
    table = batch.page_table.numpy()
    lens = batch.seq_lens.numpy()
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    G = spec.hq // spec.hkv
    if spec.mode == "sage":
        d = wl.make_sage_layer(spec, batch, 0, "cpu")
        host = {k: getattr(d, k).numpy() for k in ("q8", "sf_q", "k8", "v8", "sf_k", "sf_v", "v_mean")}
        unit, scale = "GB/s", 1e9
        per_key = spec.hkv * spec.head_dim * 2 + spec.hkv * 4 / 64
        mask = wl.make_block_mask(spec, batch, "cpu").numpy() if spec.density < 1.0 else None

        def one(i):
            r = i % spec.batch
            osg.sage_decode(host["q8"][r:r + 1], host["sf_q"][r:r + 1], host["k8"], host["v8"], host["sf_k"],
                            host["sf_v"], host["v_mean"], table[r:r + 1], lens[r:r + 1], 64,
                            block_mask=None if mask is None else mask[r:r + 1])
            L = int(lens[r])
            keys = L if mask is None else sum(min(64, L - 64 * b) for b in range(-(-L // 64)) if mask[r][b])
            return float(keys) * per_key
        per_step, what = 2, "requests"
    elif spec.mode == "extend" and args.workload == "sage_extend_prefix":
        cu = batch.cu_seqlens_q.numpy()
        d = wl.make_sage_layer(spec, batch, 0, "cpu", q_rows=int(cu[-1]))
        host = {k: getattr(d, k).numpy() for k in ("q8", "sf_q", "k8", "v8", "sf_k", "sf_v", "v_mean")}
        unit, scale = "TFLOP/s", 1e12

        def one(i):
            r, h = (i // spec.hq) % spec.batch, i % spec.hq
            hk = h // G
            q0, q1 = int(cu[r]), int(cu[r + 1])
            osg.sage_extend(host["q8"][q0:q1, h:h + 1], host["sf_q"][q0:q1, h:h + 1], np.array([0, q1 - q0]),
                            host["k8"][:, hk:hk + 1], host["v8"][:, hk:hk + 1], host["sf_k"][:, hk:hk + 1],
                            host["sf_v"][hk:hk + 1], host["v_mean"][hk:hk + 1], table[r:r + 1], lens[r:r + 1], 64)
            n = q1 - q0
            return 4.0 * spec.head_dim * (n * (int(lens[r]) - n) + n * (n + 1) // 2)
        per_step, what = 1, "(request, query head) pairs"
    elif spec.mode == "extend":
        k, v = wl.make_bf16_pools(spec, batch, 0, "cpu")
        cu = batch.cu_seqlens_q.numpy()
        q = wl.make_bf16_queries(spec, int(cu[-1]), 0, "cpu")
        kb, vb, qb = bits(k), bits(v), bits(q)
        unit, scale = "TFLOP/s", 1e12

        def one(i):
            r, h = (i // spec.hq) % spec.batch, i % spec.hq
            q0, q1 = int(cu[r]), int(cu[r + 1])
            oa.extend(qb[q0:q1, h:h + 1], np.array([0, q1 - q0]), kb[:, h // G:h // G + 1], vb[:, h // G:h // G + 1],
                      table[r:r + 1], lens[r:r + 1], spec.page_size, spec.sm_scale)
            n = q1 - q0
            return 4.0 * spec.head_dim * (n * (int(lens[r]) - n) + n * (n + 1) // 2)
        per_step, what = 2, "(request, query head) pairs"
    elif spec.mode == "fp8":
        k8, v8 = (x.numpy() for x in wl.make_fp8_pools(spec, batch, 0, "cpu"))
        qb = bits(wl.make_bf16_queries(spec, spec.batch, 0, "cpu"))
        unit, scale = "GB/s", 1e9

        def one(i):
            r = i % spec.batch
            oa.decode_fp8(qb[r:r + 1], k8, v8, wl.FP8_SCALE, wl.FP8_SCALE, table[r:r + 1], lens[r:r + 1],
                          spec.page_size, spec.sm_scale)
            return wl.decode_kv_bytes([int(lens[r])], spec.hkv, spec.head_dim, 1, spec.page_size, spec.hq, 2, 2)
        per_step, what = 2, "requests"
    else:
        k, v = wl.make_bf16_pools(spec, batch, 0, "cpu")
        q = wl.make_bf16_queries(spec, spec.batch, 0, "cpu")
        kb, vb, qb = bits(k), bits(v), bits(q)
        unit, scale = "GB/s", 1e9

        def one(i):
            r = i % spec.batch
            oa.decode(qb[r:r + 1], kb, vb, table[r:r + 1], lens[r:r + 1], spec.page_size, spec.sm_scale)
            return wl.decode_kv_bytes([int(lens[r])], spec.hkv, spec.head_dim, 2, spec.page_size, spec.hq, 2, 2)
        per_step, what = 2, "requests"
    times, units, i = [], 0.0, 0
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        u = sum(one(i + x) for x in range(per_step))
        dt = time.perf_counter() - t0
        i += per_step
        if s >= args.warmup:
            times.append(dt)
            units += u
    total = sum(times)
    value = units / total / scale if total > 0 else 0.0
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": unit, "n_gpus": 0, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * total / max(1, args.steps), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": workload_config(args.workload, spec, batch.num_slots, 1),
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{per_step} {what} of layer 0 per step, the fp64 oracle (oracle/)"},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
