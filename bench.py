"""Decode-step benchmark of the mixed-precision KV cache (one JSON line on stdout).

A step = one decode token for every sequence of the batch through every layer: per
layer, the new token's K/V is quantized and packed into the cache and decode attention
runs over it -- kvq_append_decode, one launch (a token that completes a per-channel key
group: kvq_append, then kvq_decode_attn; paged plans: kvq_append_tagged, then
kvq_decode_attn), plus the log-sum-exp merge launch when a sequence is split in two or
three (from four splits the decode launch merges its own partials).  Each step of
the decode schedule is captured once into a CUDA graph (untimed); the timed region
replays K graphs.  The dominant kernel's roofline comes from decode-only replays of the
same schedule.  Inputs are seeded synthetic tensors already resident in HBM; one step reads
every layer's cache once (larger than L2 for every workload here).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c2|c2-k8v8|c3|c4|c5|c5-alloc]
    python bench.py --impl reference ...     # the CPU oracle on a bounded sample

Under torchrun each rank runs its own replica of the workload (own seeds, no data-path
collective: weak scaling); rank 0 prints the line with the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn tokens/s and HBM GB/s (% of roofline) over mixed-precision KV, 1 B200"
FALLBACK_HBM_GBS = 6650.0


def measured_hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s pool figure)"


def kernel_source_sha256():
    import hashlib
    h = hashlib.sha256()
    for f in ("layer_wise_mixed_b200/csrc/kvq_decode.cu", "layer_wise_mixed_b200/csrc/kvq_device.cuh",
              "layer_wise_mixed_b200/csrc/kvq_internal.h"):
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()


def captured_traffic(workload_name, alg_bytes_per_launch):
    """DRAM bytes per launch of the decode kernel from the committed ncu captures (one
    block of `key: value` lines per workload, blank-line separated), scaled by algorithmic
    bytes; None when the kernel changed since the capture or no capture covers the workload."""
    p = os.path.join(ROOT, "profiles", "decode_split_traffic.txt")
    try:
        blocks, cur = [], {}
        for ln in open(p):
            if ln.startswith("#"):
                continue
            if not ln.strip():
                if cur:
                    blocks.append(cur)
                cur = {}
                continue
            if ":" in ln:
                k, v = ln.split(":", 1)
                cur[k.strip()] = v.strip()
        if cur:
            blocks.append(cur)
        sha = kernel_source_sha256()
        for kv in blocks:
            if kv.get("source_sha256") == sha and kv.get("workload") == workload_name:
                return float(kv["dram_bytes"]) / float(kv["algorithmic_bytes"]) * alg_bytes_per_launch
        return None
    except Exception:
        return None


def paged_tags(wl, n_tokens, tag="prefill", batch=None):
    """INT2/INT4 mask of a paged workload: seeded Bernoulli, or the per-tag allocation."""
    from layer_wise_mixed_b200 import inputs, tagalloc
    if wl.tag_source == "alloc":
        return tagalloc.token_mask(wl, n_tokens, tag=tag, batch=batch)
    return inputs.tags(wl, n_tokens, tag=tag, batch=batch)


def rank_workload(wl, rank, world):
    """Weak scaling: at N > 1 every rank runs its own replica of the workload on its own
    seeded sequences (the rank is part of the workload name, hence of every seed)."""
    if world <= 1:
        return wl
    import dataclasses
    return dataclasses.replace(wl, name=f"{wl.name}-rank{rank}")


def link_bound(h2d, d2h, stream, h2d_stream, d2h_stream, world, barrier, steps=16):
    """Bound of the end-to-end loop set by the host link alone: per step one pinned H2D of
    the step's input bytes and one D2H of its output bytes, issued on two copy streams at
    once (the loop's own pattern), nothing else on the GPU; CUDA events, max over ranks."""
    import torch
    hi = torch.empty(h2d // 2, dtype=torch.bfloat16).pin_memory()
    di = torch.empty(h2d // 2, dtype=torch.bfloat16, device="cuda")
    do = torch.zeros(d2h // 2, dtype=torch.bfloat16, device="cuda")
    ho = torch.empty(d2h // 2, dtype=torch.bfloat16).pin_memory()

    def run(n):
        h2d_stream.wait_stream(stream)
        d2h_stream.wait_stream(stream)
        for _ in range(n):
            with torch.cuda.stream(h2d_stream):
                di.copy_(hi, non_blocking=True)
            with torch.cuda.stream(d2h_stream):
                ho.copy_(do, non_blocking=True)
        stream.wait_stream(h2d_stream)
        stream.wait_stream(d2h_stream)

    with torch.cuda.stream(stream):
        run(3)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run(steps)
        e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world) / steps
    del hi, di, do, ho
    return {"ms_per_step": ms, "h2d_gbs": h2d / (ms / 1e3) / 1e9, "d2h_gbs": d2h / (ms / 1e3) / 1e9,
            "how": "pinned H2D of the step's input bytes and D2H of its output bytes on two copy streams at once, "
                   "nothing else running; tokens_s = batch per such step, frac = e2e / tokens_s"}


def decode_paths_entry(bytes_launch, ms_default, ms_tcgen05, peak, kernel):
    """Decode-only launch time and roofline fraction per decode path on the same schedule:
    the default (mma.sync tiles; the paged kernel for paged plans) and, where the layer
    qualifies, the tcgen05 path (kvq_set_decode_path)."""
    def one(k, ms):
        gbs = bytes_launch / (ms / 1e3) / 1e9
        return {"kernel": k, "avg_launch_us": 1e3 * ms, "hbm_gbs": gbs, "frac": gbs / peak}
    d = {"mma_sync": one(kernel, ms_default)}
    if ms_tcgen05 is not None:
        d["tcgen05"] = one("decode_umma_kernel", ms_tcgen05)
    return d


def max_over_ranks(value_ms, world):
    """Max of a per-rank time over all ranks (rank 0 reports it); plain value at N=1."""
    if world <= 1:
        return value_ms
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value_ms], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def decode_bytes(B, Hkv, G, D, L, bk, bv, kmode):
    """Algorithmic bytes of one decode-attention launch over L tokens: packed codes, fp16
    scale+zero per 32 elements, the bf16 key residual, q in and out (bf16)."""
    if kmode == 0:
        kb = (L // 32) * 32 * D * (bk + 1) / 8 + (L % 32) * D * 2
    else:
        kb = L * D * (bk + 1) / 8
    vb = L * D * (bv + 1) / 8
    return B * Hkv * (kb + vb + 2 * G * D * 2)


class ClockSampler:
    """NVML sampling of SM clock and clock-event reasons in a background thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index, period=0.02):
        self.samples = []
        self.period = period
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()
        self.t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                clk = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((clk, rs, util))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.t:
            self._stop.set()
            self.t.join()
        busy = [s for s in self.samples if s[2] > 0] or self.samples
        if not busy:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        reasons = set()
        for _, rs, _ in busy:
            for bit, name in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[0] for s in busy), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(busy)}


# ---------------------------------------------------------------- CPU oracle arm
def cpu_oracle_sample(wl, L, seqs, layers=1):
    """Time the oracle (quantize the layer's cache + fp64 attention) on `seqs` sequences
    of `layers` layers at context L; returns (seconds, tokens/s scaled to the workload)."""
    import numpy as np
    import torch

    import oracle
    from layer_wise_mixed_b200 import inputs
    t = 0.0
    for l in range(layers):
        K, V = inputs.layer_kv(wl, l, L, "cpu", batch=seqs, tag="cpu-sample")
        q = inputs.step_q(wl, l, 0, "cpu", batch=seqs)
        b16 = lambda x: x.contiguous().view(torch.int16).numpy().view(np.uint16)
        Kb, Vb, qb = b16(K), b16(V), b16(q)
        bk, bv = wl.layer_bits[l % len(wl.layer_bits)]
        t0 = time.perf_counter()
        if wl.paged:
            tg = paged_tags(wl, L, tag="cpu-sample", batch=seqs).numpy()
            oracle.paged_layer(Kb, Vb, tg, qb, wl.G, want_image=False)
        else:
            oracle.layer(Kb, Vb, qb, wl.G, bk, bv, wl.kmode, want_image=False)
        t += time.perf_counter() - t0
    step_s = t / layers * wl.num_layers * (wl.batch / seqs)
    return t, wl.batch / step_s


def run_reference(args, wl, rank):
    if rank != 0:
        return
    import oracle
    oracle.build()
    cores = os.cpu_count()
    seqs = max(1, min(wl.batch, args.ref_seqs))
    Ls = [wl.prefill + 1 + (i % max(1, wl.decode_steps)) for i in range(args.warmup + args.steps)]
    for i in range(args.warmup):
        cpu_oracle_sample(wl, Ls[i], seqs)
    tot, vals = 0.0, []
    for i in range(args.steps):
        s, v = cpu_oracle_sample(wl, Ls[args.warmup + i], seqs)
        tot += s
        vals.append(v)
    value = len(vals) / sum(1.0 / v for v in vals)
    sample = (f"per step: oracle quantize+fp64 attention of 1 of {wl.num_layers} layers for {seqs} of "
              f"{wl.batch} sequences at the step's context, scaled to the full step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * wl.batch / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(wl):
    bits = sorted(set(wl.layer_bits))
    if wl.paged:
        return {"workload": wl.name, "layers": wl.num_layers, "batch": wl.batch, "q_heads": wl.n_q_heads,
                "kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim,
                "context": f"{wl.prefill + 1}..{wl.prefill + wl.decode_steps}",
                "bits": "INT2 groups (K per-channel, V per-token) + INT4 per-token, tags " +
                        ("from the per-tag allocation at 3.0 bits (synthetic segment tag ids, seeded calibration)"
                         if wl.tag_source == "alloc" else "Bernoulli(0.5)"),
                "equivalent_bits": wl.avg_bits, "page_tokens": wl.page_tokens,
                "l2": "inputs larger than L2 (each step reads every layer's cache once)",
                "launch": "one CUDA graph per decode step (tagged append + paged decode for all layers)"}
    return {"workload": wl.name, "layers": wl.num_layers, "batch": wl.batch, "q_heads": wl.n_q_heads,
            "kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim,
            "context": f"{wl.prefill + 1}..{wl.prefill + wl.decode_steps}",
            "bits": ",".join(f"K{a}V{b}" for a, b in bits), "equivalent_bits": wl.equivalent_bits(),
            "keys": "per-channel" if wl.kmode == 0 else "per-token", "values": "per-token", "group": 32,
            "l2": "inputs larger than L2 (each step reads every layer's cache once)",
            "launch": "one CUDA graph per decode step (fused append + decode launch per layer)"}


# ---------------------------------------------------------------- GPU arm
class WorkloadRun:
    """One workload on the current device: the cache after the prefill, the decode
    schedule's inputs resident in HBM, and per decode step two CUDA graphs (captured
    once, untimed): the full step over every layer (fused append + decode launch; a
    token that completes a per-channel key group: append, then decode; paged plans:
    tagged append, then decode) and decode alone over every layer; with tcgen05=True, for
    layers the tcgen05 decode path takes (head_dim 128, G <= 8), also
    decode alone on that path."""

    def __init__(self, wl, stream, tcgen05=False):
        import numpy as np
        import torch

        from layer_wise_mixed_b200 import inputs, kvq
        self.wl, self.stream = wl, stream
        B, Hkv, Hq, D, NL = wl.batch, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.num_layers
        self.paged = paged = wl.paged
        if paged:
            all_tags = paged_tags(wl, wl.max_ctx)                  # [B, prefill + steps], shared by layers
            # the pools split at the mask's own mean bits (an allocation may land under its budget)
            plan_bits = min(wl.avg_bits, 4.0 - 2.0 * float((all_tags == 2).float().mean()))
            self.cache = kvq.Cache(NL, B, Hkv, Hq, D, wl.max_ctx, avg_bits=plan_bits)
            tags_dev = all_tags.cuda()
            self.tags_host = tags_host = all_tags.numpy()
        else:
            self.cache = kvq.Cache(NL, B, Hkv, Hq, D, wl.max_ctx, list(wl.layer_bits), kmodes=[wl.kmode] * NL)
        cache = self.cache
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for l in range(NL):
                K, V = inputs.layer_kv(wl, l, wl.prefill, "cuda")
                if paged:
                    t0 = tags_dev[:, :wl.prefill].contiguous()
                    kvq.kvq_append_tagged(cache.h, l, K, V, wl.prefill,
                                          np.ascontiguousarray(tags_host[:, :wl.prefill]), t0, stream)
                else:
                    cache.append(l, K, V)
                del K, V
        stream.synchronize()
        nsched = self.nsched = wl.decode_steps
        if paged:
            step_tags_dev = [tags_dev[:, wl.prefill + s:wl.prefill + s + 1].contiguous() for s in range(nsched)]
            step_tags_host = [np.ascontiguousarray(tags_host[:, wl.prefill + s:wl.prefill + s + 1])
                              for s in range(nsched)]
        # decode schedule inputs, resident in HBM
        self.Kn = Kn = torch.empty((nsched, NL, B, Hkv, 1, D), dtype=torch.bfloat16, device="cuda")
        self.Vn = Vn = torch.empty_like(Kn)
        self.Qn = Qn = torch.empty((nsched, NL, B, Hq, D), dtype=torch.bfloat16, device="cuda")
        for s in range(nsched):
            for l in range(NL):
                k, v = inputs.step_kv(wl, l, s, "cuda")
                Kn[s, l].copy_(k)
                Vn[s, l].copy_(v)
                Qn[s, l].copy_(inputs.step_q(wl, l, s, "cuda"))
        self.out = out = torch.empty((NL, B, Hq, D), dtype=torch.bfloat16, device="cuda")
        # one eager decode per layer before capture (kernel attributes, occupancy, status clear)
        with torch.cuda.stream(stream):
            for l in range(NL):
                cache.decode_attn(l, Qn[0, l], out[l], stream=stream)
        stream.synchronize()
        self.graphs, self.dec_graphs, self.tc_graphs, self.splits, self.Ls = [], [], [], [], []
        tc = tcgen05 and not paged and D == 128 and wl.G <= 8
        for s in range(nsched):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for l in range(NL):
                    if paged:
                        kvq.kvq_append_tagged(cache.h, l, Kn[s, l], Vn[s, l], 1, step_tags_host[s], step_tags_dev[s],
                                              stream)
                        kvq.kvq_decode_attn(cache.h, l, Qn[s, l], out[l], False, stream)
                    else:
                        kvq.kvq_append_decode(cache.h, l, Kn[s, l], Vn[s, l], Qn[s, l], out[l], False, stream)
            self.graphs.append(g)
            self.splits.append([kvq.kvq_get_num_splits(cache.h, l) for l in range(NL)])
            self.Ls.append(cache.seq_len(0))
            gd = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gd, stream=stream):
                for l in range(NL):
                    kvq.kvq_decode_attn(cache.h, l, Qn[s, l], out[l], False, stream)
            self.dec_graphs.append(gd)
            if tc:
                kvq.kvq_set_decode_path(cache.h, kvq.KVQ_DECODE_TCGEN05)
                gt = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gt, stream=stream):
                    for l in range(NL):
                        kvq.kvq_decode_attn(cache.h, l, Qn[s, l], out[l], False, stream)
                kvq.kvq_set_decode_path(cache.h, kvq.KVQ_DECODE_MMA_SYNC)
                self.tc_graphs.append(gt)
        torch.cuda.synchronize()

    def release(self):
        self.graphs, self.dec_graphs, self.tc_graphs = [], [], []

    def time_steps(self, order, warmup, barrier):
        """Device time (ms) of the full steps in `order`, after `warmup` untimed steps."""
        import torch
        stream = self.stream
        with torch.cuda.stream(stream):
            for i in range(warmup):
                self.graphs[i % self.nsched].replay()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for s in order:
                self.graphs[s].replay()
            e1.record(stream)
        barrier()
        return e0.elapsed_time(e1)

    def time_decode(self, order, min_ms=100.0, min_reps=3, tcgen05=False):
        """Decode-only graphs over the steps in `order` (the tcgen05 path's with
        tcgen05=True), replayed as a whole until at least min_ms of device time (and
        min_reps passes) are timed; returns (ms per decode launch, passes, timed ms).  Live
        CUDA events on the launching stream."""
        import torch
        stream = self.stream
        dec_graphs = self.tc_graphs if tcgen05 else self.dec_graphs
        with torch.cuda.stream(stream):
            for s in order[: min(len(order), 8)]:
                dec_graphs[s].replay()
            d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            d0.record(stream)
            for s in order:
                dec_graphs[s].replay()
            d1.record(stream)
        stream.synchronize()
        one = d0.elapsed_time(d1)
        reps = max(min_reps, int(min_ms / max(one, 1e-3)) + 1)
        with torch.cuda.stream(stream):
            d0.record(stream)
            for _ in range(reps):
                for s in order:
                    dec_graphs[s].replay()
            d1.record(stream)
        stream.synchronize()
        tot = d0.elapsed_time(d1)
        return tot / (reps * len(order) * self.wl.num_layers), reps, tot

    def decode_bytes_per_launch(self, order):
        wl = self.wl
        B, Hkv, G, D, NL = wl.batch, wl.n_kv_heads, wl.G, wl.head_dim, wl.num_layers
        if self.paged:
            # INT2 groups: 2-bit codes + fp16 scale/zero per 32 (keys and values); INT4 tokens
            # (main and pending): 4-bit codes + scale/zero; q in and out
            def paged_bytes(L):
                t = self.tags_host[:, :L]
                n2 = (t == 2).sum(1)
                g2 = (n2 // 32) * 32
                rest = L - g2
                per = g2 * D * 2 * (2 + 1) / 8 + rest * D * 2 * (4 + 1) / 8 + 2 * G * D * 2
                return float(Hkv * per.sum())
            tot = sum(paged_bytes(self.Ls[s]) for s in order for l in range(NL))
        else:
            tot = sum(decode_bytes(B, Hkv, G, D, self.Ls[s], *wl.layer_bits[l], wl.kmode)
                      for s in order for l in range(NL))
        return tot / (len(order) * NL)

    def launches(self, order):
        """Kernel launches of the steps in `order`: per layer one fused launch, or (a token
        that completes a per-channel key group; paged plans) an append and a decode launch
        (plus the tag scan of multi-token paged appends: none here); plus the merge launch
        for two or three splits."""
        wl = self.wl

        def step_launches(s, l):
            two = self.paged or (wl.kmode == 0 and self.Ls[s] % 32 == 0)
            return (2 if two else 1) + (1 if 1 < self.splits[s][l] < 4 else 0)
        return sum(step_launches(s, l) for s in order for l in range(wl.num_layers))

    def context(self, order):
        Ls = [self.Ls[s] for s in order]
        return f"{min(Ls)}..{max(Ls)}"


def reduced_workload(wl, n_layers):
    """The first n_layers layers of `wl` with the same precision mix as the full map (layers
    taken from each distinct bit pair in proportion), renumbered 0..n-1."""
    import dataclasses
    from collections import Counter
    cnt = Counter(wl.layer_bits)
    total = len(wl.layer_bits)
    bits = []
    for pair, c in sorted(cnt.items(), key=lambda x: -x[1]):
        bits += [pair] * max(1, round(n_layers * c / total))
    bits = tuple(sorted(bits, key=lambda p: wl.layer_bits.index(p)))
    return dataclasses.replace(wl, num_layers=len(bits), layer_bits=bits)


PER_CONFIG_LAYERS = {"c3": 4, "c4": 2, "c5": 2, "c5-alloc": 2, "c2-k8v8": 32, "c2": 32, "c2-k8v4": 32}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=512)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c2", choices=["c2", "c2-k8v8", "c2-k8v4", "c3", "c4", "c5", "c5-alloc"])
    ap.add_argument("--e2e-group", type=int, default=16, help="layers per H2D/D2H transfer group of the eager e2e loop")
    ap.add_argument("--e2e-mode", default="graph", choices=["graph", "eager"],
                    help="graph: per step one H2D of the step's inputs, the step's captured graph of C-ABI calls, one "
                         "D2H of its outputs; eager: per group of layers, eager C-ABI calls")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--ref-seqs", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="use only the first N layers (small ncu captures; reported in config.layers)")
    ap.add_argument("--per-config", default="c3,c4,c5",
                    help="comma list of further workloads measured after the headline (reduced layer counts with "
                         "the same precision mix; 'none' to skip)")
    ap.add_argument("--decode-ms", type=float, default=100.0,
                    help="minimum device time of the decode-only replays behind the roofline figure")
    ap.add_argument("--no-tcgen05", action="store_true",
                    help="skip the decode-only replays on the tcgen05 path (decode_paths in the JSON line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from layer_wise_mixed_b200 import configs
    wl = configs.by_name(args.workload)
    if args.layers:
        import dataclasses
        wl = dataclasses.replace(wl, num_layers=args.layers, layer_bits=wl.layer_bits[:args.layers])
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, wl, rank)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from layer_wise_mixed_b200 import kvq

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # replica per rank: its own sequences (weak scaling, no data-path collective)
    wl = rank_workload(wl, rank, world)
    B, Hkv, Hq, D, G, NL = wl.batch, wl.n_kv_heads, wl.n_q_heads, wl.head_dim, wl.G, wl.num_layers
    paged = wl.paged
    stream = torch.cuda.Stream()
    run = WorkloadRun(wl, stream, tcgen05=not args.no_tcgen05)
    cache, Kn, Vn, Qn, out, nsched = run.cache, run.Kn, run.Vn, run.Qn, run.out, run.nsched
    order = [(args.warmup + i) % nsched for i in range(args.steps)]
    peak, peak_src = measured_hbm_peak()

    # ---- timed region: K full steps; then the dominant kernel: decode-only graphs over
    # the same steps (live events), replayed for at least --decode-ms of device time ----
    sampler = ClockSampler(local)
    sampler.start()
    ms = max_over_ranks(run.time_steps(order, args.warmup, barrier), world)
    dec_launch_ms, dec_reps, dec_total_ms = run.time_decode(order, args.decode_ms)
    tc_launch_ms = run.time_decode(order, args.decode_ms, tcgen05=True)[0] if run.tc_graphs else None
    clocks = sampler.stop()
    ms_per_step = ms / args.steps
    value = world * B * args.steps / (ms / 1e3)
    launches_dec = len(order) * NL
    bytes_launch = run.decode_bytes_per_launch(order)
    achieved = bytes_launch / (dec_launch_ms / 1e3) / 1e9
    decode_paths = decode_paths_entry(bytes_launch, dec_launch_ms, tc_launch_ms, peak,
                                      "decode_paged_kernel" if paged else "decode_split_kernel")
    gpu_launches = run.launches(order)
    e2e_note = (f"per step and group of {max(1, args.e2e_group)} layers: pinned H2D of the group's K/V/q (copy stream), "
                "kvq_append_decode per layer (eager C-ABI calls, compute stream), D2H of the group's outputs "
                "(second copy stream); groups overlap")
    if paged:
        e2e_note = (f"per step and group of {max(1, args.e2e_group)} layers: pinned H2D of the group's K/V/q, kvq_decode_attn per layer "
                    "(eager C-ABI calls; the cache is not advanced), D2H of the group's outputs; groups overlap")
    if args.e2e_mode == "graph":
        e2e_note = ("per step: pinned H2D of the step's K/V/q for every layer into the step's device inputs (copy stream), "
                    "replay of the step's CUDA graph of C-ABI calls (" +
                    ("kvq_append_tagged + kvq_decode_attn" if paged else "kvq_append_decode") +
                    " per layer, captured once through the public API; compute stream), D2D of the outputs into a "
                    "double buffer and their D2H (second copy stream); consecutive steps overlap")

    # ---- e2e: public API with host buffers, H2D + D2H inside the timed region ----
    # Per step and group of CH layers (--e2e-group; fewer, larger groups issue fewer copies
    # and events: measured best at 16 of 32 layers): one H2D of the group's K|V|q (pinned
    # host, packed per layer) on a copy stream, the group's C-ABI calls on the compute stream, one D2H of
    # the group's outputs on a second copy stream (the other PCIe direction), so that
    # transfers of one group overlap the calls of another; device buffers alternate
    # between even and odd steps.
    e2e_steps = args.e2e_steps or min(args.steps, 64)
    nk, nq = B * Hkv * D, B * Hq * D                      # bf16 elements per layer
    per = 2 * nk + nq
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
    if args.e2e_mode == "eager":
        CH = max(1, args.e2e_group)
        groups = [list(range(g0, min(NL, g0 + CH))) for g0 in range(0, NL, CH)]
        hIn = torch.cat([Kn.reshape(nsched, NL, nk), Vn.reshape(nsched, NL, nk), Qn.reshape(nsched, NL, nq)],
                        dim=2).cpu().pin_memory()             # [step, layer, K|V|q]
        hO = torch.empty((NL,) + tuple(out.shape[1:]), dtype=out.dtype).pin_memory()
        dIn = torch.empty((2, NL, per), dtype=torch.bfloat16, device="cuda")
        dOut = torch.empty((2,) + tuple(out.shape), dtype=out.dtype, device="cuda")
        ev = {k: [[torch.cuda.Event() for _ in groups] for _ in range(2)] for k in ("in", "comp", "out")}
        used = [[False] * len(groups) for _ in range(2)]
        if not paged and args.e2e_mode == "eager":
            for l in range(NL):
                kvq.kvq_truncate(cache.h, l, wl.prefill)
        # raw C-ABI calls with pointers taken once (the Python wrappers cost more host time
        # per call than the transfers they would overlap)
        lib = kvq.load()
        sptr = stream.cuda_stream
        ptrs = [[(dIn[par, l].data_ptr(), dIn[par, l].data_ptr() + 2 * nk, dIn[par, l].data_ptr() + 4 * nk,
                  dOut[par, l].data_ptr()) for l in range(NL)] for par in range(2)]
        lens = [wl.prefill] * NL

        def call(l, par):
            pk, pv, pq, po = ptrs[par][l]
            if paged:
                rc = lib.kvq_decode_attn(cache.h, l, pq, po, 0, sptr)
            else:
                if lens[l] >= wl.max_ctx:
                    kvq.kvq_truncate(cache.h, l, wl.prefill)
                    lens[l] = wl.prefill
                rc = lib.kvq_append_decode(cache.h, l, pk, pv, pq, po, 0, sptr)
                lens[l] += 1
            if rc != kvq.KVQ_OK:
                raise kvq.KvqError(rc, lib.kvq_last_error().decode())

        def e2e_step(i, s):
            par = i & 1
            for gi, grp in enumerate(groups):
                l0, l1 = grp[0], grp[-1] + 1
                with torch.cuda.stream(h2d_stream):
                    if used[par][gi]:
                        h2d_stream.wait_event(ev["comp"][par][gi])     # the calls of step i - 2 read this buffer
                    dIn[par, l0:l1].copy_(hIn[s, l0:l1], non_blocking=True)
                    ev["in"][par][gi].record(h2d_stream)
                stream.wait_event(ev["in"][par][gi])
                if used[par][gi]:
                    stream.wait_event(ev["out"][par][gi])              # step i - 2's outputs are on the host
                for l in grp:
                    call(l, par)
                ev["comp"][par][gi].record(stream)
                with torch.cuda.stream(d2h_stream):
                    d2h_stream.wait_event(ev["comp"][par][gi])
                    hO[l0:l1].copy_(dOut[par, l0:l1], non_blocking=True)
                    ev["out"][par][gi].record(d2h_stream)
                used[par][gi] = True

        def drain():
            for par in range(2):
                for gi in range(len(groups)):
                    if used[par][gi]:
                        stream.wait_event(ev["out"][par][gi])

    if args.e2e_mode == "graph":
        # the step's inputs land in the device tensors its graph reads (Kn/Vn/Qn[s], one
        # per step of the schedule); outputs alternate between two device buffers for the D2H
        hK, hV, hQ = Kn.cpu().pin_memory(), Vn.cpu().pin_memory(), Qn.cpu().pin_memory()
        out2 = torch.empty((2,) + tuple(out.shape), dtype=out.dtype, device="cuda")
        hO2 = torch.empty((2,) + tuple(out.shape), dtype=out.dtype).pin_memory()
        gev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "comp", "out")}
        gused = [False, False]

        def e2e_step(i, s):
            par = i & 1
            with torch.cuda.stream(h2d_stream):
                Kn[s].copy_(hK[s], non_blocking=True)
                Vn[s].copy_(hV[s], non_blocking=True)
                Qn[s].copy_(hQ[s], non_blocking=True)
                gev["in"][par].record(h2d_stream)
            stream.wait_event(gev["in"][par])
            run.graphs[s].replay()
            if gused[par]:
                stream.wait_event(gev["out"][par])           # step i - 2's outputs are on the host
            out2[par].copy_(out, non_blocking=True)
            gev["comp"][par].record(stream)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(gev["comp"][par])
                hO2[par].copy_(out2[par], non_blocking=True)
                gev["out"][par].record(d2h_stream)
            gused[par] = True

        def drain():
            for par in range(2):
                if gused[par]:
                    stream.wait_event(gev["out"][par])
    e2e_first = args.warmup + args.steps   # continue the schedule where the timed steps ended
    with torch.cuda.stream(stream):
        for i in range(3):
            e2e_step(i, (e2e_first + i) % nsched)
        drain()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        h2d_stream.wait_stream(stream)
        d2h_stream.wait_stream(stream)
        for i in range(e2e_steps):
            e2e_step(3 + i, (e2e_first + 3 + i) % nsched)
        drain()
        f1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world)
    e2e_value = world * B * e2e_steps / (e2e_ms / 1e3)
    h2d = NL * per * 2
    d2h = out.numel() * 2
    link = link_bound(h2d, d2h, stream, h2d_stream, d2h_stream, world, barrier)
    link["tokens_s"] = world * B / (link["ms_per_step"] / 1e3)
    link["frac"] = e2e_value / link["tokens_s"]
    status = kvq.kvq_device_status(cache.h, stream)
    head_cfg = workload_config(wl)
    head_cfg["context"] = run.context(order)
    head_cfg["schedule"] = f"{wl.prefill + 1}..{wl.prefill + wl.decode_steps}"
    traffic = captured_traffic(wl.name, bytes_launch)
    head_splits = sorted(set(x for s in order for x in run.splits[s]))
    run.release()
    del run, cache
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    # ---- further workloads (rank 0 of a 1-GPU run): the long-context maps and the paged
    # cache, reduced to a few layers with the same precision mix; step throughput scaled to
    # the full layer count, the decode kernel's roofline per launch ----
    per_config = {}
    wanted = [] if args.per_config in ("", "none") else [x for x in args.per_config.split(",") if x]
    if world == 1:
        for name in wanted:
            full = configs.by_name(name)
            wc = reduced_workload(full, PER_CONFIG_LAYERS.get(name, 2))
            r = WorkloadRun(wc, stream, tcgen05=not args.no_tcgen05)
            ordc = list(range(r.nsched))
            smp = ClockSampler(local)
            smp.start()
            ms_c = r.time_steps(ordc, 3, barrier)
            dl_ms, dl_reps, _ = r.time_decode(ordc, args.decode_ms)
            tl_ms = r.time_decode(ordc, args.decode_ms, tcgen05=True)[0] if r.tc_graphs else None
            clk = smp.stop()
            bl = r.decode_bytes_per_launch(ordc)
            ach = bl / (dl_ms / 1e3) / 1e9
            st = kvq.kvq_device_status(r.cache.h, stream)
            per_config[name] = {
                "workload": full.name, "layers_measured": wc.num_layers, "layers_full": full.num_layers,
                "bits_measured": ",".join(f"K{a}V{b}" for a, b in wc.layer_bits) if not wc.paged else "INT2/INT4",
                "batch": wc.batch, "timed_context": r.context(ordc), "steps": len(ordc),
                "tokens_per_s": wc.batch / (ms_c / len(ordc) * full.num_layers / wc.num_layers / 1e3),
                "step_ms_per_layer": ms_c / len(ordc) / wc.num_layers,
                "hbm_gbs_decode": ach, "frac": ach / peak, "avg_launch_us": 1e3 * dl_ms,
                "algorithmic_bytes_per_launch": bl, "decode_replays": dl_reps,
                "traffic": captured_traffic(full.name, bl),
                "kernel": "decode_paged_kernel" if wc.paged else "decode_split_kernel",
                "splits": sorted(set(x for s in ordc for x in r.splits[s])), "clocks": clk, "device_status": st,
                "decode_paths": decode_paths_entry(bl, dl_ms, tl_ms, peak,
                                                   "decode_paged_kernel" if wc.paged else "decode_split_kernel"),
                "how": (f"{wc.num_layers} of {full.num_layers} layers with the full map's precision mix; tokens/s = "
                        "batch / (step time scaled to the full layer count); decode GB/s = algorithmic bytes / "
                        "CUDA-event time of decode-only graph replays")}
            r.release()
            del r
            torch.cuda.synchronize()
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_cpu, v_cpu = 0.0, []
        L_mid = wl.prefill + max(1, wl.decode_steps // 2)
        while t_cpu < 10.0:
            s_, v_ = cpu_oracle_sample(wl, L_mid, max(1, min(B, args.ref_seqs)))
            t_cpu += s_
            v_cpu.append(v_)
        cpu = {"value": len(v_cpu) / sum(1 / v for v in v_cpu), "unit": "tokens/s", "cores": os.cpu_count(),
               "kind": "oracle",
               "sample": (f"{len(v_cpu)} x (quantize + fp64 attention of 1 layer, {min(B, args.ref_seqs)} of {B} "
                          f"sequences, context {L_mid}), {t_cpu:.1f} s CPU, scaled to a full step")}
        # the same sample on one thread (about 3 s)
        import oracle
        threads = oracle.set_threads(0)
        oracle.set_threads(1)
        t1, v1 = 0.0, []
        while t1 < 3.0:
            s_, v_ = cpu_oracle_sample(wl, L_mid, max(1, min(B, args.ref_seqs)))
            t1 += s_
            v1.append(v_)
        oracle.set_threads(threads)
        cpu["single_thread"] = {"value": len(v1) / sum(1 / v for v in v1), "unit": "tokens/s", "cores": 1}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f16*f16->f32 (codes exact in f16), f32 quantizer",
                "data": "synthetic (seeded normal K/V/Q, outlier key channels; no weights or datasets)",
                "config": head_cfg,
                "hbm_gbs_decode": achieved,
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                             "frac": achieved / peak, "traffic": traffic,
                             "kernel": "decode_paged_kernel" if wl.paged else "decode_split_kernel",
                             "peak_source": peak_src, "avg_launch_us": 1e3 * dec_launch_ms,
                             "algorithmic_bytes_per_launch": bytes_launch,
                             "decode_region": {"replays_of_timed_steps": dec_reps, "ms": dec_total_ms,
                                               "launches": dec_reps * launches_dec}},
                "cpu_baseline": cpu,
                "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                        "steps": e2e_steps, "how": e2e_note,
                        "host_link_gbs": {"h2d": h2d * e2e_steps / (e2e_ms / 1e3) / 1e9,
                                          "d2h": d2h * e2e_steps / (e2e_ms / 1e3) / 1e9},
                        "link_bound": link},
                "gpu_launches": gpu_launches, "clocks": clocks, "device_status": status,
                "splits": head_splits,
                "decode_paths": decode_paths,
                "per_config": per_config}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
