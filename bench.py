#!/usr/bin/env python
"""Benchmark of the decode-step hybrid sparse + linear attention on B200.

One step = for every layer of the workload: one decode (block scores, top-k,
gather, exact softmax part, Taylor linear part by subtraction, merge) and one
append (the new token's cache row; the evicted token's fold into the linear
state and block statistics happens in the next decode), issued as one
hyb_attn_decode_append call: one launch of the fused decode kernel per layer,
consecutive layers chained with programmatic dependent launch.

Prints one JSON line (rank 0).  ``--impl reference`` times the fp64 CPU oracle
on a bounded sample of the same workload instead.

Multi-GPU: one process per GPU (torchrun); every rank runs its own copy of the
workload's units (independent batches; no collective on the data path) and the
step time is the max over ranks ("scaling": "weak").
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_FLUSH_BYTES = 512 << 20
METRIC = "hybrid decode-attn steps/s and achieved HBM GB/s (% of peak) at 32K-256K ctx"
DEFAULT_WORKLOAD = "llama8b_32layers_b8_32k"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-sample-seconds", type=float, default=12.0)
    ap.add_argument("--layers", type=int, default=None,
                    help="override the workload's layer count (smaller instances for profiling)")
    ap.add_argument("--mode", default="decode", choices=["decode", "spec", "prefill", "strided"],
                    help="decode: one decode + append per layer and step; spec: hyb_attn_decode_chunk of "
                         "--chunk draft tokens per layer and step; prefill: hyb_attn_append_chunk of --chunk "
                         "tokens, then one decode, per layer and step; strided: hyb_attn_decode_strided "
                         "(stride --chunk, the workload's top-k among the other blocks), then one append, "
                         "per layer and step")
    ap.add_argument("--chunk", type=int, default=4)
    return ap.parse_args()


# ----------------------------------------------------------------------------- ranks

def rank_workload(w, rank: int):
    """Each rank runs its own replica of the workload's units (weak scaling): the
    same shapes, its own seeded data, no collective on the data path."""
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + rank) if rank else w


def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's time (all ranks take this step, in the same order)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_steps_per_s(ms_per_step_max: float, world: int) -> float:
    """Whole-job throughput: every rank completes one step of its own units per
    ms_per_step_max."""
    return world * 1e3 / ms_per_step_max


# ----------------------------------------------------------------------------- bytes model

def algorithmic_bytes(w, T):
    """Bytes one decode must move per (layer, b, kv head) at length T, and the
    append's bytes per unit (the method's minimum: selected/exact tokens, block
    statistics, linear state, q and out; no unselected token)."""
    d, G = w.head_dim, w.group
    per = w.bytes_per_unit(T)
    decode = sum(per.values())
    # cache write of the new token, read of the evicted token, and the write-back
    # of the state the decode already reads: H, zk, zv, n, and one block's mean /
    # variance row
    append = (2 * d * 2) + (2 * d * 2) + d * d * 4 + 2 * d * 4 + 4 + 2 * d * 4
    return decode, append


def spec_bytes(w, T: int, n: int, union_blocks: float):
    """Bytes per (layer, b, kv head) of n draft rows decoded together (rows at
    lengths T .. T + n - 1) with their appends: what the rows share is counted
    once -- the block statistics of the last row's blocks, the sinks and the
    union of the rows' windows, the linear state, and the union of the rows'
    selected blocks (`union_blocks`, measured) -- plus every row's q and output;
    the appends write n cache rows, read the n tokens they evict and write the
    state back once."""
    d, G = w.head_dim, w.group
    Tl = T + n - 1
    sinks = min(w.n_sink, Tl)
    window = Tl - max(w.n_sink, Tl - w.window) if Tl > w.n_sink else 0
    exact = sinks + window + min(w.evicted(Tl), union_blocks * w.block_size)
    dec = w.n_blocks(Tl) * 2 * d * 4 + exact * d * 2 * 2 + (d * d + 2 * d + 1) * 4 + n * G * d * 6
    app = n * 4 * d + n * 4 * d + d * d * 4 + 2 * d * 4 + 4 + 2 * 2 * d * 4
    return dec, app


def step_bytes_model(w, mode: str, chunk: int, T: int, union_blocks=None):
    """(decode bytes, all bytes, flush L2?) of one step at length about T: every
    layer with its own budget; prefill: the chunk's rows and evicted tokens, the
    state written back once, one decode; spec: the chunk's draft rows decoded
    together (spec_bytes, with the measured union of their selections per layer;
    without it, the bytes of one decode per row)."""
    step_dec = step_bytes = 0
    for l in range(w.layers):
        if w.head_budgets or mode == "strided":
            wl = w.for_layer(l)
            for h in range(w.n_kv_heads):
                wh = wl.for_head(h)
                if mode == "strided":  # the union selection, and the statistics read again by its launch
                    nb = wh.n_blocks(T)
                    wh = dataclasses.replace(wh, top_k=nb // chunk + min(wh.top_k, nb - nb // chunk))
                dec_b, app_b = algorithmic_bytes(wh, T)
                if mode == "strided":
                    dec_b += wh.n_blocks(T) * 2 * wh.head_dim * 4
                step_dec += w.batch * dec_b
                step_bytes += w.batch * (dec_b + app_b)
            continue
        if mode == "spec" and union_blocks is not None:
            dec_b, app_b = spec_bytes(w.for_layer(l), T, chunk, union_blocks[l])
            step_dec += w.units_per_layer * dec_b
            step_bytes += w.units_per_layer * (dec_b + app_b)
            continue
        dec_b, app_b = algorithmic_bytes(w.for_layer(l), T)
        if mode == "prefill":
            d = w.head_dim
            app_b = chunk * 8 * d + (d * d + 2 * d + 1) * 4 + (-(-chunk // w.block_size) + 1) * 2 * d * 4
        per_step = chunk if mode == "spec" else 1  # decodes per layer and step
        step_dec += w.units_per_layer * dec_b * per_step
        step_bytes += w.units_per_layer * (dec_b + app_b) * per_step
    flush = step_bytes < 4 * 126e6      # the step's data would otherwise stay in L2
    return step_dec, step_bytes, flush


KERNEL_SOURCES = {"fused": ("k_fused.cu", "k_common.cuh", "hyb_device.cuh", "hyb_internal.h"),
                  "multi": ("k_multi.cu", "k_common.cuh", "hyb_device.cuh", "hyb_internal.h")}


def kernel_sources_hash(kernel: str = "fused") -> str:
    import hashlib
    csrc = os.path.join(ROOT, "hybrid_sparse_linear_decode_b200", "csrc")
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profile_name(workload: str, mode: str = "decode", chunk: int = 1) -> str:
    """The committed ncu summary of the launch the bench's roofline is about:
    the fused decode kernel, or (spec mode) the multi-query kernel at the
    chunk's group size."""
    if mode == "spec":
        return f"multi_decode_{workload}_rows{chunk}.md"
    return f"fused_decode_{workload}.md"


def measured_traffic(workload: str, mode: str = "decode", chunk: int = 1):
    """DRAM bytes of one launch of the dominant kernel from the committed ncu
    summary of this workload, if the kernel's sources are unchanged since that
    capture (else None)."""
    import re
    if mode not in ("decode", "spec"):  # several kernels per step: no single launch's capture applies
        return None
    prof = os.path.join(ROOT, "profiles", profile_name(workload, mode, chunk))
    if not os.path.exists(prof):
        return None
    text = open(prof).read()
    mh = re.search(r"kernel_sources_sha256_16:\s*([0-9a-f]{16})", text)
    mt = re.search(r"traffic_bytes_per_launch:\s*(\d+)", text)
    if not (mh and mt):
        return None
    return int(mt.group(1)) if kernel_sources_hash("multi" if mode == "spec" else "fused") == mh.group(1) else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- native arm

class Bench:
    def __init__(self, w, n_steps, device, mode="decode", chunk=1):
        import torch
        import syngen.device as SD
        from syngen import host as SH
        from hybrid_sparse_linear_decode_b200 import HybridAttentionLayer, make_config
        self.w, self.device = w, device
        self.n_steps = n_steps
        self.mode, self.chunk = mode, (chunk if mode != "decode" else 1)
        n_app = self.n_steps * (self.chunk if mode in ("spec", "prefill") else 1)  # strided: chunk is the stride

        def cfg_of(l):  # the layer's own top-k and window when budgets vary by layer (or by KV head)
            wl = w.for_layer(l)
            heads = [wl.for_head(h) for h in range(w.n_kv_heads)]
            top_k = max(wh.top_k for wh in heads)
            if self.mode == "strided":  # the selection row holds the strided blocks and the top-k
                nb = w.n_blocks(w.T0 + n_app)
                top_k = nb // self.chunk + min(top_k, nb - nb // self.chunk)
            hw = [wh.window for wh in heads] if w.head_budgets else None
            hk = [wh.top_k for wh in heads] if w.head_budgets else None
            return make_config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block_size, w.n_sink,
                               min(wh.window for wh in heads), top_k, w.T0 + n_app, head_window=hw, head_top_k=hk)

        ws_bytes = max(HybridAttentionLayer.workspace_bytes(cfg_of(l)) for l in range(w.layers))
        self.workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=device)   # shared: one stream
        self.layers, self.app_k, self.app_v, self.q = [], [], [], []
        n_q = min(self.n_steps, 8)
        for l in range(w.layers):
            L = HybridAttentionLayer(cfg_of(l), device, workspace=self.workspace)
            tb = SD.DeviceTables(w, l, L.device)
            SD.fill_kv(w, tb, L.k_cache, L.v_cache, 0, w.T0)
            shp = (w.batch, w.n_kv_heads, n_app, w.head_dim)
            ak = torch.empty(shp, dtype=torch.bfloat16, device=device)
            av = torch.empty(shp, dtype=torch.bfloat16, device=device)
            SD.fill_kv(w, tb, ak, av, w.T0, w.T0 + n_app, t_out0=w.T0)
            if self.mode == "prefill":  # per step a chunk, contiguous [step][B][Hkv][chunk][d]
                shp5 = (w.batch, w.n_kv_heads, self.n_steps, self.chunk, w.head_dim)
                self.app_k.append(ak.view(shp5).permute(2, 0, 1, 3, 4).contiguous())
                self.app_v.append(av.view(shp5).permute(2, 0, 1, 3, 4).contiguous())
            else:  # per appended token, contiguous [token][B][Hkv][d]
                self.app_k.append(ak.permute(2, 0, 1, 3).contiguous())
                self.app_v.append(av.permute(2, 0, 1, 3).contiguous())
            del ak, av
            qs = []
            for s in range(n_q):
                qb = SH.q_bits(w, l, s)
                qs.append(torch.from_numpy(qb.view("int16")).to(device).view(torch.bfloat16))
            if self.mode == "spec":  # one chunk of draft queries [chunk][B][Hq][d], reused every step
                qs = [torch.stack([qs[i % n_q] for i in range(self.chunk)]).contiguous()]
            self.q.append(qs)
            L.init(w.T0)
            self.layers.append(L)
        self.out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32, device=device)
        self.out_chunk = torch.empty((self.chunk, w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32,
                                     device=device)
        torch.cuda.synchronize()
        self.step_idx = 0

    def step(self):
        s = self.step_idx
        n = self.chunk
        for l, L in enumerate(self.layers):
            q = self.q[l][s % len(self.q[l])]
            if self.mode == "spec":
                L.decode_chunk(q, self.app_k[l][s * n:(s + 1) * n], self.app_v[l][s * n:(s + 1) * n],
                               out=self.out_chunk)
            elif self.mode == "strided":
                L.decode_strided(q, self.w.for_layer(l).top_k, n, out=self.out)
                L.append(self.app_k[l][s], self.app_v[l][s])
            elif self.mode == "prefill":
                L.append_chunk(self.app_k[l][s], self.app_v[l][s])
                L.decode(q, out=self.out)
            else:
                L.decode_append(q, self.app_k[l][s], self.app_v[l][s], out=self.out)
        self.step_idx += 1

    def launches_per_step(self):
        """Kernels per step: one fused decode launch per layer (the append's
        cache write and the fold of the previous evictions ride in it); spec:
        one multi-query launch per group of 4, then 2, then 1 draft rows;
        prefill: the chunk's cache write, the dense fold of the tokens it
        evicted (5 or more) and one decode; strided: the selection (which
        scores the block holding the previous step's eviction from its rows
        folded on the fly), the decode (which folds that eviction into the
        state) and the append's cache write."""
        n = self.chunk
        groups = n // 4 + (n % 4) // 2 + (n % 2)
        per = {"decode": 1, "spec": groups, "prefill": 2 + (self.chunk >= 5), "strided": 3}[self.mode]
        return per * len(self.layers)

    def union_blocks(self):
        """Spec mode: the rows of one step decoded with their selections kept;
        per layer, the mean over units of the number of distinct blocks the
        rows selected (consumes one step, before any timing)."""
        import torch
        w, n, s = self.w, self.chunk, self.step_idx
        res = []
        for l, L in enumerate(self.layers):
            wl = w.for_layer(l)
            sel = torch.full((n, w.batch, w.n_kv_heads, wl.top_k), -1, dtype=torch.int32, device=self.device)
            L.decode_chunk(self.q[l][s % len(self.q[l])], self.app_k[l][s * n:(s + 1) * n],
                           self.app_v[l][s * n:(s + 1) * n], out=self.out_chunk, sel_out=sel)
            a = sel.cpu().numpy().reshape(n, -1, wl.top_k)
            res.append(float(np.mean([len(set(a[:, u].ravel().tolist()) - {-1}) for u in range(a.shape[1])])))
        self.step_idx += 1
        return res


def run_native(args, rank, world):
    import torch
    from syngen import configs as C
    torch.cuda.set_device(rank % torch.cuda.device_count())
    device = torch.device("cuda", torch.cuda.current_device())
    w = rank_workload(C.get_workload(args.workload, **({"layers": args.layers} if args.layers else {})), rank)
    K, Wm = args.steps, args.warmup
    mode, chunk = args.mode, (args.chunk if args.mode != "decode" else 1)
    Kk = min(K, 20) if mode == "decode" else 0  # steps of the pass timing each launch on its own
    Ke = 0 if (args.no_e2e or mode != "decode") else min(K, 20)  # steps of the end-to-end pass
    Kp = 1 if mode == "spec" else 0  # the step that measures the rows' union of selected blocks
    b = Bench(w, Kp + Wm + K + Kk + Ke, device, mode, chunk)
    union = b.union_blocks() if mode == "spec" else None
    T_mid = w.T0 + (Kp + Wm + K // 2) * chunk
    step_dec, step_bytes, flush = step_bytes_model(w, mode, chunk, T_mid, union)
    scratch = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device) if flush else None

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(Wm):
        b.step()
        if flush:
            scratch.zero_()
    torch.cuda.synchronize()

    # ---- timed region: K steps, device time with CUDA events, max over ranks
    stream = torch.cuda.current_stream()
    clk = ClockSampler(torch.cuda.current_device())
    clk.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    if flush:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        for i in range(K):
            evs[i][0].record(stream)
            b.step()
            evs[i][1].record(stream)
            scratch.zero_()
        torch.cuda.synchronize()
        total_ms = sum(e0.elapsed_time(e1) for e0, e1 in evs)
    else:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(K):
            b.step()
        e1.record(stream)
        torch.cuda.synchronize()
        total_ms = e0.elapsed_time(e1)
    barrier()
    clocks = clk.stop()
    total_ms = max_over_ranks(total_ms, world, device)
    ms_per_step = total_ms / K
    steps_s = 1e3 / ms_per_step

    # ---- the launch on its own: events around each layer's launch, chaining off
    ka, kb_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    kern_ms, n_kern = 0.0, 0
    pool = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in b.layers]
            for _ in range(Kk)]
    for i in range(Kk):
        for l, L in enumerate(b.layers):
            e0, e1 = pool[i][l]
            e0.record(stream)
            e1.record(stream)
            L.set_timing_events(e0, e1)
        b.step()
        for L in b.layers:
            L.set_timing_events(None, None)
        if flush:
            scratch.zero_()
    torch.cuda.synchronize()
    for i in range(Kk):
        for e0, e1 in pool[i]:
            kern_ms += e0.elapsed_time(e1)
            n_kern += 1
    isolated_ms = kern_ms / n_kern if n_kern else None
    # In the timed region the step is exactly one launch of the fused kernel per
    # layer, back to back: its average duration there is the step time over the
    # launches, and its algorithmic bytes those of one layer's decode + append.
    n_launch = b.launches_per_step()
    launch_ms = ms_per_step / n_launch
    launch_bytes = step_bytes // n_launch
    hbm_peak, peak_kind = peaks()
    achieved = launch_bytes / (launch_ms * 1e-3) / 1e9
    isolated = launch_bytes / (isolated_ms * 1e-3) / 1e9 if isolated_ms else None
    step_gbs = step_bytes / (ms_per_step * 1e-3) / 1e9

    # ---- e2e through the whole-step host entry point: per step one copy of every
    # layer's q / k / v in from pinned host memory, every layer's decode +
    # append, one copy of every layer's output back (hyb_attn_step_layers_host)
    e2e = None
    if Ke > 0:
        import hybrid_sparse_linear_decode_b200 as H
        ctxs = [L.ctx for L in b.layers]
        nst = H.hyb_attn_step_layers_staging_bytes(ctxs)
        staging = torch.empty(nst, dtype=torch.uint8, device=device)
        s0 = b.step_idx
        assert s0 + Ke <= b.n_steps
        hin, per_layer_in = [], None
        for i in range(Ke):  # each step's inputs, layer after layer: q, k, v (bf16 bytes), pinned
            s = s0 + i
            parts = []
            for l in range(len(b.layers)):
                parts += [b.q[l][s % len(b.q[l])].reshape(-1), b.app_k[l][s].reshape(-1), b.app_v[l][s].reshape(-1)]
            flat = torch.cat(parts).cpu()
            per_layer_in = flat.numel() * 2
            hin.append(flat.pin_memory())
        hout = torch.empty(len(b.layers) * w.batch * w.n_q_heads * w.head_dim, dtype=torch.float32).pin_memory()
        sh = stream.cuda_stream
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Ke)]
        for i in range(Ke):
            evs[i][0].record(stream)
            H.hyb_attn_step_layers_host(ctxs, hin[i].data_ptr(), hout.data_ptr(), staging.data_ptr(), nst, sh)
            evs[i][1].record(stream)
            b.step_idx += 1
            if flush:
                scratch.zero_()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(sum(a.elapsed_time(c) for a, c in evs) / Ke, world, device)
        h2d = per_layer_in
        d2h = hout.numel() * 4
        e2e = {"value": round(aggregate_steps_per_s(e2e_ms, world), 3), "unit": "steps/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5),
               "call": "hyb_attn_step_layers_host (one copy in, every layer's decode + append, one copy out)"}

    status = 0
    for L in b.layers:
        status |= L.status()
    result = {
        "metric": METRIC,
        "value": round(aggregate_steps_per_s(ms_per_step, world), 3),
        "unit": "steps/s",
        "n_gpus": world,
        "steps": K,
        "warmup": Wm,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded counter-based generator; no dataset, no weights)",
        "config": workload_config(w, mode, chunk, world, flush),
        "attention_tokens_per_s": round(world * steps_s * w.batch * chunk, 3),
        "context_tokens_per_s": round(world * steps_s * w.batch * w.layers * T_mid, 1),
        "achieved_gbs_step": round(step_gbs, 1),
        "pct_of_hbm_peak_step": round(100 * step_gbs / hbm_peak, 2),
        "bytes_per_step": step_bytes,
        **({"union_selected_blocks_per_unit": [round(u, 2) for u in union],
            "bytes_model": "draft rows decoded together: shared reads counted once, the union of the rows' "
                           "selected blocks as measured"} if union is not None else {}),
        "roofline": {"bound": "hbm",
                     "kernel": ("the multi-query decode kernel: one layer's draft rows decoded + appended together"
                                if mode == "spec" else
                                "one layer's launches, averaged: the strided selection, the decode, the append"
                                if mode == "strided" else
                                "one layer's launches, averaged: the chunk's cache write, the dense fold, the decode"
                                if mode == "prefill" else "the fused decode kernel: one layer's decode + append (one launch)"),
                     "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "peak_kind": peak_kind,
                     "traffic": measured_traffic(w.name, mode, chunk), "bytes_per_launch": launch_bytes,
                     "decode_bytes_per_launch": step_dec // n_launch,
                     "avg_launch_us": round(launch_ms * 1e3, 3),
                     "isolated_launch_us": round(isolated_ms * 1e3, 3) if isolated_ms else None,
                     "isolated_frac": round(isolated / hbm_peak, 4) if isolated else None},
        "e2e": e2e,
        "gpu_launches": b.launches_per_step() * K,
        "clocks": clocks,
        "device_status": status,
    }
    return result


# ----------------------------------------------------------------------------- oracle (CPU) arm
#
# The fp64 oracle is timed on whole units of the workload in worker processes,
# one single-threaded worker per host core (BLAS limited to one thread), so that
# "cores" is the number of threads that actually ran.  Workers are started with
# the spawn method (never forked from a process that has used CUDA) and import
# neither torch nor the CUDA library.  A full step holds more units than host
# memory does (32 layers x 64 units at 32K is ~137 GB in fp64), so the workers
# time decode + append pairs on copies of a few units and the step time is
# extrapolated from them.

def _oracle_unit_inputs(w, unit_id: int, max_appends: int):
    """Inputs of unit `unit_id` of the workload (layers cycle first, so that
    units of different per-layer budgets and head scales are sampled): its keys
    and values for [0, T0 + max_appends), the step-0 query of its group, and its
    (window, top_k): its layer's, or its KV head's when the budgets vary by head."""
    from syngen import host as SH
    layer, j = unit_id % w.layers, unit_id // w.layers
    wl = w.for_layer(layer)
    b, h = divmod(j % (w.batch * w.n_kv_heads), w.n_kv_heads)
    tb = SH.LayerTables(wl, layer)
    q_all = SH.bf16_bits_to_f64(SH.q_bits(wl, layer, 0))
    K, V = SH.kv_f64(wl, tb, b, h, 0, w.T0 + max_appends)
    wh = wl.for_head(h)
    return K, V, np.ascontiguousarray(q_all[b, h * w.group:(h + 1) * w.group]), wh.window, wh.top_k


def _oracle_sample_unit(e, seconds: float, stride=None):
    """Decode + append pairs on one unit for about `seconds` of timed work; when
    its prepared tokens are used up it starts again from T0 (the rebuild is not
    timed).  With `stride`, the decode takes the strided selection: the block
    scores from the unit's statistics, the strided blocks plus the top-k of the
    others, then the decode given that selection (which scores the blocks once
    more, as the unit's decode always does).  Returns (pairs, decode seconds,
    append seconds)."""
    O = e["O"]
    t_dec = t_app = 0.0
    n = 0
    while t_dec + t_app < seconds:
        if e["pos"] >= e["n_app"]:
            e["u"], e["pos"] = e["fresh"](), 0
        u, pos = e["u"], e["pos"]
        t0 = time.perf_counter()
        if stride is None:
            u.decode(e["q"])
        else:
            mu, var = u.stats()
            nb = mu.shape[0]
            sc = O.block_scores(e["q"], mu, var, u.scale) if nb else np.zeros(0)
            u.decode(e["q"], sel=O.select_blocks_strided(sc, u.k, stride))
        t1 = time.perf_counter()
        u.append(e["K"][e["T0"] + pos], e["V"][e["T0"] + pos])
        t2 = time.perf_counter()
        t_dec += t1 - t0
        t_app += t2 - t1
        e["pos"] = pos + 1
        n += 1
    if n == 0:
        raise RuntimeError("oracle sample timed no unit")
    return n, t_dec, t_app


def _oracle_worker(conn, spec: dict):
    """Worker process: one BLAS thread; its unit built once from the inputs in
    shared memory, then one sample per request until it receives None."""
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    sys.path.insert(0, ROOT)
    from multiprocessing import shared_memory
    import oracle as O
    shm = shared_memory.SharedMemory(name=spec["shm"])
    T, d, G = spec["T"], spec["d"], spec["G"]
    buf = np.ndarray((2 * T * d + G * d,), dtype=np.float64, buffer=shm.buf)
    K = buf[:T * d].reshape(T, d)
    V = buf[T * d:2 * T * d].reshape(T, d)
    q = buf[2 * T * d:].reshape(G, d).copy()
    T0 = spec["T0"]

    def fresh():
        return O.OracleUnit(K[:T0], V[:T0], spec["S"], spec["W"], spec["Bk"], spec["k"], spec["scale"],
                            capacity=T)

    e = {"fresh": fresh, "u": fresh(), "K": K, "V": V, "q": q, "T0": T0, "n_app": T - T0, "pos": 0, "O": O}
    conn.send("ready")
    try:
        while True:
            msg = conn.recv()
            if msg is None:
                break
            conn.send(_oracle_sample_unit(e, *msg))   # (seconds, stride or None)
    finally:
        del K, V, buf, e
        shm.close()
        conn.close()


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class OraclePool:
    """Single-threaded oracle worker processes, one per host core (bounded by
    host memory).  The parent generates the inputs of a few distinct units once
    into shared memory; every worker builds its own oracle unit from one of them
    and times decode + append pairs on it (the oracle's cost does not depend on
    the values)."""

    def __init__(self, w, max_appends: int = 256):
        import multiprocessing as mp
        from multiprocessing import shared_memory
        try:
            import psutil
            avail = psutil.virtual_memory().available
        except Exception:
            avail = 16 << 30
        d, G = w.head_dim, w.group
        T = w.T0 + max_appends
        n_units_total = w.layers * w.units_per_layer
        n_distinct = min(n_units_total, 2 if w.T0 <= 65536 else 1)
        per_worker = 2 * T * d * 8 + 2 * (w.n_blocks(T) + 1) * d * 8   # the oracle unit's K, V copy, block sums
        by_mem = max(1, int((0.5 * avail - n_distinct * 2 * T * d * 8) // per_worker))
        self.workers = max(1, min(host_cores(), by_mem))
        self.w = w
        self.units = n_distinct
        self.shms, specs = [], []
        for i in range(n_distinct):
            K, V, q, win, k = _oracle_unit_inputs(w, i, max_appends)
            shm = shared_memory.SharedMemory(create=True, size=(2 * T * d + G * d) * 8)
            buf = np.ndarray((2 * T * d + G * d,), dtype=np.float64, buffer=shm.buf)
            buf[:T * d] = K.reshape(-1)
            buf[T * d:2 * T * d] = V.reshape(-1)
            buf[2 * T * d:] = q.reshape(-1)
            del buf
            self.shms.append(shm)
            specs.append({"shm": shm.name, "T": T, "T0": w.T0, "d": d, "G": G, "S": w.n_sink, "W": win,
                          "Bk": w.block_size, "k": k, "scale": 1 / math.sqrt(d)})
        ctx = mp.get_context("spawn")
        self.conns, self.procs = [], []
        for i in range(self.workers):
            a, b = ctx.Pipe()
            p = ctx.Process(target=_oracle_worker, args=(b, specs[i % n_distinct]), daemon=True)
            p.start()
            self.conns.append(a)
            self.procs.append(p)
        for c in self.conns:
            if c.recv() != "ready":
                raise RuntimeError("oracle worker failed to start")

    def sample(self, seconds: float, mode: str = "decode", chunk: int = 1):
        """All workers time `seconds` of decode + append pairs at once.  Returns
        (seconds per full step, extrapolated from the timed units; pairs timed)."""
        for c in self.conns:
            c.send((seconds, chunk if mode == "strided" else None))
        res = [c.recv() for c in self.conns]
        rate = 0.0   # unit steps per second, all workers together
        pairs = 0
        for n, td, ta in res:
            dd, aa = td / n, ta / n
            per_unit_step = {"decode": dd + aa, "spec": chunk * (dd + aa), "prefill": chunk * aa + dd,
                             "strided": dd + aa}[mode]
            rate += 1.0 / per_unit_step
            pairs += n
        units_per_step = self.w.layers * self.w.units_per_layer
        return units_per_step / rate, pairs

    def describe(self, pairs: int, mode: str, chunk: int) -> str:
        w = self.w
        what = {"decode": "decode + append", "spec": f"{chunk} x (decode + append)",
                "prefill": f"{chunk} appends + decode",
                "strided": f"strided selection (stride {chunk}) + decode + append"}[mode]
        return (f"extrapolated from {self.units} units: {pairs} timed decode + append pairs on whole "
                f"(layer, b, kv-head) units at {w.T0}+ tokens, {self.workers} single-threaded worker processes "
                f"at once, each with its own copy of one of the {self.units} units; a step = {what} per unit, "
                f"x{w.layers * w.units_per_layer} units")

    def close(self):
        for c in self.conns:
            try:
                c.send(None)
            except Exception:
                pass
        for p in self.procs:
            p.join(timeout=10)
            if p.is_alive():
                p.terminate()
        for shm in self.shms:
            shm.close()
            shm.unlink()
        self.shms = []


def workload_config(w, mode: str, chunk: int, world: int, flush: bool) -> dict:
    """The `config` object of the JSON line (both arms)."""
    return {
        "workload": w.name, "layers": w.layers, "batch": w.batch, "n_q_heads": w.n_q_heads,
        "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "context_T0": w.T0, "block": w.block_size,
        "sinks": w.n_sink, "window": w.window, "top_k": w.top_k,
        **({"layer_budgets_k_W": [list(x) for x in w.layer_budgets]} if w.layer_budgets else {}),
        **({"head_budgets_k_W": [list(x) for x in w.head_budgets]} if w.head_budgets else {}),
        "l2": "flushed between timed steps (512 MB write)" if flush else "step data >> L2 (no flush)",
        "parallelism": f"replicas x{world} (independent units per GPU)",
        **({"mode": mode, "stride": chunk} if mode == "strided" else {"mode": mode, "chunk": chunk} if mode != "decode" else {}),
    }


def run_reference(args, rank, world):
    from syngen import configs as C
    overrides = {"layers": args.layers} if args.layers else {}
    w = C.get_workload(args.workload, **overrides)
    mode, chunk = args.mode, (args.chunk if args.mode != "decode" else 1)
    pool = OraclePool(w)
    try:
        per = args.cpu_sample_seconds / max(1, args.steps)
        for _ in range(args.warmup):
            pool.sample(min(0.1, per), mode, chunk)
        samples, pairs = [], 0
        t_wall = time.perf_counter()
        for _ in range(args.steps):
            s, n = pool.sample(per, mode, chunk)
            samples.append(s)
            pairs += n
        t_wall = time.perf_counter() - t_wall
    finally:
        pool.close()
    ms = 1e3 * statistics.mean(samples)
    v = 1e3 / ms
    _, _, flush = step_bytes_model(w, mode, chunk, w.T0)
    desc = pool.describe(pairs, mode, chunk)
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based generator; no dataset, no weights)",
        "config": workload_config(w, mode, chunk, world, flush),
        "cpu_baseline": {"value": round(v, 6), "unit": "steps/s", "cores": pool.workers, "kind": "oracle",
                         "sample": desc, "extrapolated_from_units": pool.units},
        "e2e": {"value": round(v, 6), "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "extrapolated": f"each step is a {per:.3f} s sample of {pool.units} units timed on {pool.workers} host "
                        f"cores, scaled to the workload's {w.layers * w.units_per_layer} units; wall time of the "
                        f"timed samples {t_wall:.2f} s",
    }


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", rank)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_native(args, rank, world)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        from syngen import configs as C
        overrides = {"layers": args.layers} if args.layers else {}
        w = C.get_workload(args.workload, **overrides)
        mode, chunk = args.mode, (args.chunk if args.mode != "decode" else 1)
        pool = OraclePool(w)
        try:
            pool.sample(0.1, mode, chunk)   # warm numpy in every worker
            s, pairs = pool.sample(args.cpu_sample_seconds, mode, chunk)
        finally:
            pool.close()
        res["cpu_baseline"] = {"value": round(1.0 / s, 6), "unit": "steps/s", "cores": pool.workers,
                               "kind": "oracle", "sample": pool.describe(pairs, mode, chunk),
                               "extrapolated_from_units": pool.units}
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
