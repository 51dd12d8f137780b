"""Benchmark: MoBA block-sparse attention prefill on B200, one JSON line.

One step is the whole hot path over one batch of the workload: key pooling, gate
scores + top-k + dispatch lists, and block-sparse attention with the merge
(moba_pool_keys -> moba_select_topk -> moba_attn_fwd), inputs resident in HBM.
`value` is attended TFLOP/s (4 d |J_i| summed over rows, heads and batch, divided by
the device time of the step); tokens/s, per-stage and per-pass times, the dense-causal
comparators (torch SDPA and this library's own kernel with a window >= N) and the
roofline of the dominant kernel ride along.  `e2e` measures the same through the
binding's host-buffer entry (host->device copies of q, k, v and device->host copies of
out, lse inside the timed region).  The default workload is the 1M-token prefill; the
32K, hybrid 64K and sliding-window 16K workloads are measured after it in the same run
and reported under "workloads".  `--impl reference` times the fp64 CPU oracle instead.

Multi-GPU (torchrun): every rank runs its own copy of the workload (the method
shards over batch / kv-head groups with no exchange): weak scaling, no collective on
the data path; the timed region is bracketed by barriers and the max over ranks is
reported.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "block-sparse attn prefill TFLOPS & tokens/s vs dense causal, % of roofline"
UNIT = "TFLOP/s (attended)"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="moba1m", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--extra-workloads", default="gqa32k,hybrid64k,swa16k",
                    help="comma-separated workloads measured after the main one (rank 0 "
                         "reports them under 'workloads'); empty for none")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-comparators", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ multi-rank

def max_over_ranks(value: float, device) -> float:
    """The largest of every rank's value (one all-reduce; identity without a group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job rate: every rank processed units_per_rank in at most max_ms."""
    return units_per_rank * world / (max_ms * 1e-3)


def source_digest() -> str:
    """sha256 over the library sources: ties a stored ncu traffic figure to the
    kernels it was measured on."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_long_prefill_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(f.encode() + b"\0" + fh.read())
    return h.hexdigest()


def stored_traffic(workload: str, kernel: str = None):
    """DRAM bytes per launch of `kernel` (or of the whole attention stage) from the
    committed ncu summary, or None when the kernels changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    rec = d.get(workload)
    if not rec or rec.get("sources_sha256") != source_digest():
        return None
    if kernel is None:
        return rec.get("attention_dram_bytes_per_step")
    return rec.get("per_kernel_bytes", {}).get(kernel)


# ------------------------------------------------------------------ accounting

def attended_pairs_moba(idx: torch.Tensor, w: workloads.Workload) -> int:
    """Sum over rows, heads and batch of |J_i| for the blocks in idx (own block causal,
    past blocks whole) unioned with the causal window.  Row r of idx sits at key
    position q_off + r (q_off > 0 for a chunked prefill)."""
    B = w.block
    i = w.q_off + torch.arange(w.nq, device=idx.device)
    c = i // B
    own = (i % B) + 1
    past = ((idx >= 0) & (idx < c[None, None, :, None])).sum(-1)  # [b, h, N]
    total = own.sum().item() * w.batch * w.hq + int(past.sum().item()) * B
    if w.window > 0:
        # Window keys in blocks the row did not select.
        extra = 0
        for blk_off in range(1, (w.window + B - 1) // B + 1):
            blk = c - blk_off
            ok = blk >= 0
            lo = torch.clamp(i - w.window + 1, min=0)
            start = torch.maximum(blk * B, lo)
            end = torch.minimum(blk * B + B - 1, i)
            cnt = torch.clamp(end - start + 1, min=0) * ok
            sel = (idx == blk[None, None, :, None]).any(-1)
            extra += int((cnt[None, None, :] * (~sel)).sum().item())
        total += extra
    return int(total)


def attended_pairs_swa(w: workloads.Workload) -> int:
    i = np.arange(w.seqlen, dtype=np.int64)
    return int(np.minimum(i + 1, w.window).sum()) * w.batch * w.hq


def pass_work_moba(idx: torch.Tensor, w: workloads.Workload) -> dict:
    """Algorithmic work of each moba_attn_fwd pass, summed over all query chunks:
    attended FLOPs (4*d per (query, key) pair) of the past-block pass (whole selected
    past blocks) and of the own-block pass (causal own block plus window tail keys),
    and the bytes the merge pass must move (topk partial rows and log-sum-exps read,
    block choices read, the output row and its log-sum-exp written)."""
    B, N = w.block, w.nq
    i = w.q_off + torch.arange(N, device=idx.device)   # key positions of the rows
    c = i // B
    past = int(((idx >= 0) & (idx < c[None, None, :, None])).sum().item()) * B
    own = int(((i % B) + 1).sum().item()) * w.batch * w.hq
    if w.window > 0:
        own += attended_pairs_moba(idx, w) - own - past  # window keys outside the choices
    rowcount = w.batch * w.hq * N
    merge_bytes = rowcount * (w.topk * (w.d * 2 + 4) + w.topk * 4 + w.d * 2 + 4)
    return {"past_block_pass": 4.0 * w.d * past, "own_block_pass": 4.0 * w.d * own,
            "merge_pass": merge_bytes}


def dense_pairs(w: workloads.Workload) -> int:
    """Causal pairs of the query rows (positions q_off .. seqlen - 1)."""
    Nk, off = w.seqlen, w.q_off
    return (Nk * (Nk + 1) // 2 - off * (off + 1) // 2) * w.batch * w.hq


# --------------------------------------------------------------------- clocks

def physical_gpu(local: int) -> str:
    """The nvidia-smi id (index or UUID) of CUDA device `local` of this process."""
    vis = [x.strip() for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    return vis[local] if local < len(vis) else str(local)


_REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
            ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))


class ClockSampler:
    """Samples the SM clock, its maximum and the active clock-event reasons of one GPU
    while the timed region runs.  NVML (the library nvidia-smi reads) is polled every
    few milliseconds from a thread, so that even a timed region of tens of
    milliseconds is covered; `mark_start()` / `mark_stop()` bracket the region and
    only samples inside it are summarised.  Without NVML it falls back to nvidia-smi
    at its shortest period.  Read-only: nothing about the GPU is changed."""

    def __init__(self, device: int, period_s: float = 0.002):
        self.device = device
        self.period = period_s
        self.samples = []          # (t, sm_mhz, max_mhz, reasons bitmask, power_w)
        self.t0 = self.t1 = None
        self._stop = False
        self._thread = None
        self._smi = None
        self._path = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        try:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId_v2(bus.encode())
        except Exception:
            pass
        try:
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(props.uuid)).encode())
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(int(physical_gpu(self.device)))

    def _poll(self, nv, h):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self._stop:
            try:
                self.samples.append((time.perf_counter(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     mx, int(get_reasons(h)), nv.nvmlDeviceGetPowerUsage(h) / 1000.0))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        try:
            import threading
            nv, h = self._nvml_handle()
            self._thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self._thread.start()
            deadline = time.perf_counter() + 2.0
            while not self.samples and time.perf_counter() < deadline:
                time.sleep(0.001)
        except Exception:
            self._thread = None
            self._start_smi()
        return self

    def _start_smi(self):
        try:
            import tempfile
            fd, self._path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self._smi = subprocess.Popen(
                ["nvidia-smi", "-i", physical_gpu(self.device),
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self._path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(1.0)
        except Exception:
            self._smi = None

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_stop(self):
        self.t1 = time.perf_counter()

    def __exit__(self, *exc):
        self._stop = True
        if self._thread is not None:
            self._thread.join(timeout=2)
        if self._smi is not None:
            self._smi.terminate()
            try:
                self._smi.wait(timeout=5)
            except Exception:
                self._smi.kill()

    def _smi_samples(self):
        out = []
        if not self._path or not os.path.exists(self._path):
            return out
        names = [n for n, _ in _REASONS[:4]]
        with open(self._path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm, mx = float(parts[0]), float(parts[1])
                except ValueError:
                    continue
                mask = 0
                for (n, bit), v in zip(_REASONS[:4], parts[4:8]):
                    if v.lower().startswith("active"):
                        mask |= bit
                out.append((None, sm, mx, mask, None))
        os.unlink(self._path)
        return out

    def summary(self):
        if self._thread is not None:
            inside = [x for x in self.samples
                      if self.t0 is not None and self.t1 is not None and self.t0 <= x[0] <= self.t1]
            source = "nvml"
        else:
            inside = self._smi_samples()
            source = "nvidia-smi"
        if not inside:
            return None
        reasons = sorted({n for x in inside for n, bit in _REASONS if x[3] & bit})
        pw = [x[4] for x in inside if x[4] is not None]
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": inside[0][2],
                "sm_mhz_min": min(x[1] for x in inside), "reasons": reasons,
                "power_w_median": round(statistics.median(pw), 1) if pw else None,
                "samples": len(inside), "source": source}


# ------------------------------------------------------------------- our arm

def layout_chunks(w: workloads.Workload) -> int:
    """Query chunks moba_attn_fwd runs (the partials of one chunk stay below 4 GiB)."""
    per_row = (w.topk if w.topk > 1 else 0) * (w.d * 2 + 4) * w.batch * w.hq
    if per_row == 0 or per_row * w.nq <= (4 << 30):
        return 1
    chunk_rows = max(128, ((4 << 30) // per_row) // 128 * 128)
    return math.ceil(w.nq / chunk_rows)


def launches_per_step(w: workloads.Workload) -> int:
    """Library kernels one step launches: pool, gate, scatter (+ a scan launch when the
    general gate runs: the tensor-core gate's last CTA writes the list offsets itself),
    and per query chunk: past-block pass, own-block pass, merge (only the own-block
    pass when topk = 1)."""
    if w.kind != "moba":
        return 1
    tc_gate = -(-w.seqlen // w.block) <= 256 and w.topk - 1 < 32 and w.gate == "mean"
    if w.gate == "static":
        sel = 1 + (2 if w.topk > 1 else 0)       # static gate, scan, scatter
    else:
        sel = 2 + ((1 if tc_gate else 2) if w.topk > 1 else 0)
    return sel + layout_chunks(w) * (3 if w.topk > 1 else 1)


def measure(w, steps, warmup, rank, world, device, seed, full=True, cpu_leg=True,
            comparators=True):
    """Times `steps` steps of workload w (after `warmup` untimed ones) and returns the
    result dict.  full: also the end-to-end host-buffer leg; cpu_leg: the CPU oracle
    baseline (rank 0, one GPU); comparators: the dense comparators (rank 0)."""
    import block_sparse_long_prefill_b200 as moba
    from block_sparse_long_prefill_b200 import MobaPrefill

    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream()
    q, k, v = workloads.make_inputs(w, seed=seed + rank)
    if w.q_off:
        q = q[:, :, w.q_off:].contiguous()  # chunked prefill: the last nq query rows
    qd, kd, vd = q.to(device), k.to(device), v.to(device)
    if full:
        qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    del q, k, v
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)  # > 126 MB L2

    nchunks = layout_chunks(w) if w.kind == "moba" else 1
    if w.kind == "moba":
        runner = MobaPrefill(w.batch, w.hq, w.hkv, w.nq, w.d, w.block, w.topk, w.window,
                             device=device, kv_len=w.seqlen)

        def stages():
            if w.gate == "minmax":
                moba.moba_pool_keys_minmax(kd, w.block, out=runner.kbar_split)
                yield "pool"
                moba.moba_select_topk_minmax(qd, runner.kbar_split, w.block, w.topk, w.seqlen,
                                             runner.workspace, runner.idx)
            elif w.gate == "static":
                yield "pool"  # no pooled keys
                moba.moba_select_static(w.batch, w.hq, w.hkv, w.nq, w.d, w.block, w.topk, w.sink,
                                        runner.workspace, kv_len=w.seqlen, idx=runner.idx)
            else:
                moba.moba_pool_keys(kd, w.block, runner.kbar, runner.kbar_split)
                yield "pool"
                moba.moba_select_topk_chunk(qd, runner.kbar_split, w.block, w.topk, w.seqlen,
                                            runner.workspace, runner.idx)
            yield "select"
            moba.moba_attn_fwd_chunk(qd, kd, vd, runner.idx, w.block, w.topk, runner.workspace,
                                     w.window, out=runner.out, lse=runner.lse)
            yield "attention"
        out_t, lse_t = runner.out, runner.lse
    else:
        out_t = torch.empty_like(qd)
        lse_t = torch.empty(w.batch, w.hq, w.seqlen, dtype=torch.float32, device=device)

        def stages():
            moba.swa_attn_fwd(qd, kd, vd, w.window, out=out_t, lse=lse_t)
            yield "attention"

    # Events recorded by moba_attn_fwd before its first kernel and after each launch
    # (every pass of every query chunk), so that each kernel is timed over all of its
    # launches on the stream it runs on.
    chunk_passes = []
    if w.kind == "moba":
        chunk_passes = (["past_block_pass", "own_block_pass", "merge_pass"] if w.topk > 1
                        else ["own_block_pass"])
    pass_seq = chunk_passes * nchunks
    pass_evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(pass_seq) + 1)]
    per_pass = {n: 0.0 for n in chunk_passes}

    def step_timed():
        evs = [torch.cuda.Event(enable_timing=True)]
        evs[0].record(stream)
        names = []
        for name in stages():
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            evs.append(e)
            names.append(name)
        return evs, names

    for _ in range(warmup):
        for _ in stages():
            pass
    torch.cuda.synchronize()
    assert moba.device_status() == 0

    pairs = attended_pairs_moba(runner.idx, w) if w.kind == "moba" else attended_pairs_swa(w)
    flops = 4.0 * w.d * pairs

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    per_stage = {}
    total_ms = 0.0
    if pass_seq:
        moba.set_pass_events(pass_evs)
    with ClockSampler(torch.cuda.current_device()) as clk:
        clk.mark_start()
        for _ in range(steps):
            flush.zero_()
            evs, names = step_timed()
            torch.cuda.synchronize()
            total_ms += evs[0].elapsed_time(evs[-1])
            for a, b_, n in zip(evs[:-1], evs[1:], names):
                per_stage.setdefault(n, []).append(a.elapsed_time(b_))
            for a, b_, n in zip(pass_evs[:-1], pass_evs[1:], pass_seq):
                per_pass[n] += a.elapsed_time(b_) / steps
        clk.mark_stop()
    torch.cuda.synchronize()
    if pass_seq:
        moba.set_pass_events(None)
    total_ms = max_over_ranks(total_ms, device)
    if world > 1:
        torch.distributed.barrier()
    assert moba.device_status() == 0
    assert torch.isfinite(out_t.float()).all().item(), "non-finite output"
    ms = total_ms / steps
    tflops_total = weak_scaling_rate(flops, world, ms) / 1e12
    tokens = weak_scaling_rate(w.batch * w.nq, world, ms)

    hbm, tc_peak, tc_sus, peak_kind = peaks()
    stage_ms = {n: sum(v_) / len(v_) for n, v_ in per_stage.items()}
    attn_ms = stage_ms["attention"]
    achieved = flops / (attn_ms * 1e-3) / 1e12
    extra = {}
    kname = f"attn_fwd_kernel<{w.d}, 0>"
    if w.kind == "moba":
        work = pass_work_moba(runner.idx, w)
        passes = {}
        for n in chunk_passes:
            t = per_pass[n] * 1e-3
            rec = {"ms": round(per_pass[n], 4), "launches": nchunks}
            if n == "merge_pass":
                gbs = work[n] / t / 1e9
                rec.update({"bytes": work[n], "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4)})
            else:
                tf = work[n] / t / 1e12
                rec.update({"flops": work[n], "tflops": round(tf, 2), "frac": round(tf / tc_peak, 4)})
            passes[n] = rec
        extra["passes"] = passes
        extra["attention_stage"] = {"ms": round(attn_ms, 4), "tflops": round(achieved, 2),
                                    "frac": round(achieved / tc_peak, 4),
                                    "note": "whole moba_attn_fwd call: all passes, all query chunks"}
        dom = max((n for n in chunk_passes if n != "merge_pass"), key=lambda n: per_pass[n])
        kname = f"attn_fwd_kernel<{w.d}, {1 if dom == 'past_block_pass' else 0}>"
        traffic = stored_traffic(w.name, kname)
        roofline = {"bound": "tensor", "achieved": passes[dom]["tflops"], "peak": tc_peak,
                    "unit": "TFLOP/s", "frac": passes[dom]["frac"],
                    "traffic": traffic,
                    "kernel": f"{kname} ({dom.replace('_', ' ')}; {nchunks} launches per step, "
                              "one per query chunk)",
                    "work": "4*d FLOPs per attended (query, key) pair of the pass, all launches",
                    "peak_kind": f"bf16 dense burst, {peak_kind}",
                    "frac_of_sustained": round(passes[dom]["tflops"] / tc_sus, 4) if tc_sus else None}
    else:
        traffic = stored_traffic(w.name, kname)
        roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": tc_peak,
                    "unit": "TFLOP/s", "frac": round(achieved / tc_peak, 4),
                    "traffic": traffic,
                    "kernel": f"{kname} (swa_attn_fwd: one launch)",
                    "work": "4*d FLOPs per attended (query, key) pair",
                    "peak_kind": f"bf16 dense burst, {peak_kind}"}
    if w.kind == "moba":
        sel_ms = stage_ms["pool"] + stage_ms["select"]
        n_entries = int(((runner.idx >= 0).sum().item()) - w.batch * w.hq * w.nq)
        sel_bytes = 2 * w.batch * w.hq * w.nq * w.topk * 4 + 2 * n_entries * 4
        if w.gate != "static":  # the keys and the queries are read once
            sel_bytes += w.batch * w.hkv * w.seqlen * w.d * 2 + w.batch * w.hq * w.nq * w.d * 2
        extra["selection"] = {"ms": round(sel_ms, 4), "bytes": sel_bytes,
                              "gbs": round(sel_bytes / (sel_ms * 1e-3) / 1e9, 1),
                              "frac_hbm": round(sel_bytes / (sel_ms * 1e-3) / 1e9 / hbm, 4)}

    # ---------------------------------------------------------------- backward
    if (w.kind == "moba" and w.gate == "mean" and w.window == 0 and not w.q_off
            and w.d in (64, 128)):
        bws_bytes = moba.bwd_workspace_size(w.batch, w.hq, w.hkv, w.nq, w.d, w.block, w.topk)
        if bws_bytes <= (16 << 30):
            extra["backward"] = time_backward(w, qd, kd, vd, runner, flush, stream, steps,
                                              warmup, flops / (4.0 * w.d), tc_peak, seed + rank)

    # ---------------------------------------------------------------- e2e (host buffers)
    e2e = None
    if full:
        out_h = torch.empty(out_t.shape, dtype=out_t.dtype, pin_memory=True)
        lse_h = torch.empty(lse_t.shape, dtype=lse_t.dtype, pin_memory=True)
        e2e_ms = 0.0
        # The MoBA prefill from host buffers goes through MobaPrefillHost, which overlaps
        # the copies of one KV-head group with the kernels of the previous one; the
        # variants (chunks, other gates) copy in, run and copy out in sequence.
        host = None
        if w.kind == "moba" and w.gate == "mean" and not w.q_off:
            host = moba.MobaPrefillHost(w.batch, w.hq, w.hkv, w.seqlen, w.d, w.block, w.topk,
                                        w.window, device=device)
        for it in range(warmup + steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            if host is not None:
                host(qh, kh, vh, out_h, lse_h)
            else:
                qd.copy_(qh, non_blocking=True)
                kd.copy_(kh, non_blocking=True)
                vd.copy_(vh, non_blocking=True)
                for _ in stages():
                    pass
                out_h.copy_(out_t, non_blocking=True)
                lse_h.copy_(lse_t, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            if it >= warmup:
                e2e_ms += e0.elapsed_time(e1)
        if host is not None:
            # The pipelined result is the device path's (checked on the last step).
            assert torch.equal(out_h, out_t.cpu()) and torch.equal(lse_h, lse_t.cpu()), "e2e mismatch"
            del host
        e2e_ms = max_over_ranks(e2e_ms, device) / steps
        h2d = (qh.numel() + kh.numel() + vh.numel()) * 2
        d2h = out_h.numel() * 2 + lse_h.numel() * 4
        e2e = {"value": round(flops * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
               "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "path": "MobaPrefillHost (pinned host buffers, KV-head groups pipelined)"
                       if (w.kind == "moba" and w.gate == "mean" and not w.q_off)
                       else "copies in, the step, copies out"}
        del out_h, lse_h

    # ---------------------------------------------------------------- comparators
    comps = {}
    if comparators and rank == 0:
        comps = dense_comparators(w, qd, kd, vd, flush, stream, ms, steps, tc_peak)

    cpu = None
    if full and cpu_leg and rank == 0 and world == 1:
        cpu = cpu_baseline(w, seed, target_s=12.0, tensors=None if w.q_off else (qh, kh, vh))

    clocks = clk.summary()
    line = {"value": round(tflops_total, 2), "ms_per_step": round(ms, 4),
            "config": {"workload": w.name, "batch": w.batch, "hq": w.hq, "hkv": w.hkv,
                       "seq_len": w.seqlen, "q_len": w.nq, "gate": w.gate, "d": w.d,
                       "block": w.block, "topk": w.topk,
                       "window": w.window, "parallelism": f"replicas x{world}" if world > 1 else "1 gpu",
                       "l2": "flushed between timed steps (256 MB write)"},
            "tokens_per_s": round(tokens, 1), "attended_flops_per_step": flops,
            "stages_ms": {k_: round(v_, 4) for k_, v_ in stage_ms.items()},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step(w) * steps, "clocks": clocks}
    line.update(extra)
    line.update(comps)
    return line


def time_backward(w, qd, kd, vd, runner, flush, stream, steps, warmup, pairs, tc_peak, seed):
    """moba_attn_bwd over the forward's choices: one call (prep, dQ, dK/dV and dQ merge
    kernels) timed with CUDA events, L2 flushed between calls.  Algorithmic work is
    10 d FLOPs per attended pair (the five products of softmax attention's backward);
    the kernels execute 14 d (the dQ pass recomputes S and dP)."""
    import block_sparse_long_prefill_b200 as moba
    do = workloads.make_grad(w, seed).to(qd.device)
    bws = torch.empty(moba.bwd_workspace_size(w.batch, w.hq, w.hkv, w.nq, w.d, w.block, w.topk),
                      dtype=torch.uint8, device=qd.device)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)

    def call():
        moba.moba_attn_bwd(qd, kd, vd, runner.out, runner.lse, do, runner.idx, w.block, w.topk,
                           runner.workspace, dq=dq, dk=dk, dv=dv, bwd_workspace=bws)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(steps):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b_ = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b_.record(stream)
        torch.cuda.synchronize()
        tot += a.elapsed_time(b_)
    assert moba.device_status() == 0
    ms = tot / steps
    flops = 10.0 * w.d * pairs
    del do, bws, dq, dk, dv
    return {"ms": round(ms, 4), "flops": flops, "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
            "frac": round(flops / (ms * 1e-3) / 1e12 / tc_peak, 4),
            "executed_flops": 14.0 * w.d * pairs, "launches": 4,
            "work": "10*d FLOPs per attended pair (dQ, dK, dV of softmax attention)"}


def dense_comparators(w, qd, kd, vd, flush, stream, moba_ms, steps, tc_peak):
    """Dense causal attention on the same inputs: this library's own kernel (sliding
    window >= N) and torch SDPA (a library call).  Problems above a PFLOP are timed
    once, after a warm-up on their first 8192 rows."""
    import torch.nn.functional as F

    import block_sparse_long_prefill_b200 as moba
    dflops = 4.0 * w.d * dense_pairs(w)
    big = dflops > 1e15
    reps = 1 if big else max(3, steps // 4)

    def timeit(fn, warm):
        for _ in range(1 if big else 2):
            warm()
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(reps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b_ = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b_.record(stream)
            torch.cuda.synchronize()
            tot += a.elapsed_time(b_)
        return tot / reps

    def sl(t):  # the first 8192 rows (warm-up of the big problems)
        return t[:, :, :8192] if big else t

    own_out = torch.empty_like(qd)
    own_lse = torch.empty(w.batch, w.hq, w.nq, dtype=torch.float32, device=qd.device)
    od_ms = timeit(lambda: moba.swa_attn_fwd_chunk(qd, kd, vd, w.seqlen, out=own_out, lse=own_lse),
                   lambda: moba.swa_attn_fwd(sl(qd), sl(kd), sl(vd), w.seqlen))
    del own_out, own_lse
    comps = {"dense_causal_own_kernel": {"ms": round(od_ms, 4), "reps": reps,
                                         "tflops": round(dflops / (od_ms * 1e-3) / 1e12, 2),
                                         "frac_of_peak": round(dflops / (od_ms * 1e-3) / 1e12
                                                               / tc_peak, 4)}}
    if not w.q_off:
        # torch's is_causal aligns the queries with the first keys, so it times whole
        # prefills only.
        G = w.hq // w.hkv
        kr = kd.repeat_interleave(G, dim=1) if G > 1 else kd
        vr = vd.repeat_interleave(G, dim=1) if G > 1 else vd
        sd_ms = timeit(lambda: F.scaled_dot_product_attention(qd, kr, vr, is_causal=True),
                       lambda: F.scaled_dot_product_attention(sl(qd), sl(kr), sl(vr), is_causal=True))
        del kr, vr
        comps["dense_causal_sdpa"] = {"ms": round(sd_ms, 4), "reps": reps,
                                      "tflops": round(dflops / (sd_ms * 1e-3) / 1e12, 2),
                                      "speedup_of_moba": round(sd_ms / moba_ms, 3)}
    return comps


def run_ours(args, rank, world, device):
    w = workloads.WORKLOADS[args.workload]
    main = measure(w, args.steps, args.warmup, rank, world, device, args.seed,
                   full=not args.no_e2e, cpu_leg=not args.no_cpu_baseline,
                   comparators=not args.no_comparators)
    line = {"metric": METRIC, "value": main.pop("value"), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": main.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) q,k,v; per-block key offsets; no dataset)"}
    line.update(main)
    extras = [x for x in args.extra_workloads.split(",") if x and x != w.name]
    if extras:
        torch.cuda.empty_cache()
        line["workloads"] = {}
        for name in extras:
            we = workloads.WORKLOADS[name]
            r = measure(we, max(5, min(args.steps, 10)), args.warmup, rank, world, device,
                        args.seed, full=False, comparators=not args.no_comparators)
            for key in ("cpu_baseline", "e2e"):
                r.pop(key, None)
            r["steps"] = max(5, min(args.steps, 10))
            line["workloads"][name] = r
            torch.cuda.empty_cache()
    return line


# ------------------------------------------------------------ oracle timing

def cpu_baseline(w: workloads.Workload, seed: int, target_s: float, tensors=None):
    """Times the fp64 oracle on this workload: the full key pooling plus selection and
    attention for a seeded sample of query rows (all heads), sized to about target_s
    seconds; reports the attended TFLOP/s extrapolated to the whole workload.
    ``tensors``: the workload's (q, k, v) host tensors when already drawn."""
    import oracle

    q, k, v = tensors if tensors is not None else workloads.make_inputs(w, seed)
    rng = np.random.default_rng(seed + 2000)
    N = w.nq  # query rows: positions q_off .. seqlen - 1

    def run(nrows):
        rows = (w.q_off + np.sort(rng.choice(N, size=nrows, replace=False))).astype(np.int32)
        t0 = time.perf_counter()
        if w.kind == "moba":
            if w.gate == "static":
                t1 = time.perf_counter()
                idx = oracle.select_static(w.seqlen, w.block, w.topk, w.sink, rows, w.batch, w.hq)
            elif w.gate == "minmax":
                kmax, kmin = oracle.pool_minmax(k, w.block)
                t1 = time.perf_counter()
                s = oracle.minmax_scores(q, kmax, kmin, w.block, rows)
                idx, _ = oracle.select_topk(s, w.seqlen, w.block, w.topk, rows)
            else:
                kbar = oracle.pool_keys(k, w.block)
                t1 = time.perf_counter()
                s = oracle.gate_scores(q, kbar, w.block, rows)
                idx, _ = oracle.select_topk(s, w.seqlen, w.block, w.topk, rows)
            oracle.attention(q, k, v, mode=oracle.MODE_MOBA, block=w.block, topk=w.topk, idx=idx,
                             window=w.window, rows=rows)
            t2 = time.perf_counter()
            i = rows.astype(np.int64)
            c = i // w.block
            pairs_rows = int(((i % w.block) + 1 + np.minimum(w.topk - 1, c) * w.block).sum()) * w.batch * w.hq
            return t1 - t0, t2 - t1, pairs_rows
        oracle.swa(q, k, v, window=w.window, rows=rows)
        t2 = time.perf_counter()
        pairs_rows = int(np.minimum(rows.astype(np.int64) + 1, w.window).sum()) * w.batch * w.hq
        return 0.0, t2 - t0, pairs_rows

    probe = min(N, 32)
    tp, ta, _ = run(probe)
    per_row = max(ta / probe, 1e-6)
    nrows = int(min(N, max(probe, target_s / per_row)))
    tp, ta, pairs_rows = run(nrows)
    full_s = tp + ta * N / nrows
    pairs = attended_pairs_swa(w) if w.kind == "swa" else None
    if pairs is None:
        i = w.q_off + np.arange(N, dtype=np.int64)
        pairs = int(((i % w.block) + 1 + np.minimum(w.topk - 1, i // w.block) * w.block).sum()) * w.batch * w.hq
    flops = 4.0 * w.d * pairs
    return {"value": flops / full_s / 1e12, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"full key pooling + {nrows} of {N} query rows x {w.batch * w.hq} heads "
                      f"(seeded); whole-workload time extrapolated by rows: {full_s:.1f} s",
            "sample_seconds": round(tp + ta, 2)}


def run_reference(args, rank, world):
    """The oracle on the host cores as the reference arm (rank 0 only)."""
    w = workloads.WORKLOADS[args.workload]
    if rank != 0:
        return None
    per_step = []
    last = None
    # The inputs are drawn once; every step times the oracle on its own row sample.
    tensors = workloads.make_inputs(w, args.seed)
    for it in range(args.warmup + args.steps):
        last = cpu_baseline(w, args.seed + it, target_s=3.0, tensors=tensors)
        if it >= args.warmup:
            per_step.append(last["value"])
    value = statistics.median(per_step)
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "batch": w.batch, "hq": w.hq, "hkv": w.hkv,
                       "seq_len": w.seqlen, "q_len": w.nq, "gate": w.gate, "d": w.d,
                       "block": w.block, "topk": w.topk,
                       "window": w.window},
            "cpu_baseline": {**last, "value": value},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    line = run_ours(args, rank, world, torch.device("cuda", local))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
