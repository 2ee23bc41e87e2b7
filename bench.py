"""Benchmark of the B200 fused attention forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one call of the whole hot path (fa_fwd: tile scheduling, TMA
staging, both tcgen05 contractions, online softmax, epilogue) over one batch
of synthetic input of the named workload (default: the LLaMA-13B-shaped
self-attention B=1, H=40, N=8192, d=128, bf16, causal, BSND).  Inputs are
resident in HBM when the timed region starts; enough input sets rotate that
a step never starts with its own inputs in L2: at least two, and at least
twice the 126 MB L2 in total (16 sets of 17 MB for the cross-attention
workload; the default workload's 336 MB sets exceed L2 on their own).

Prints ONE JSON line on rank 0.  With N > 1 (torchrun), every rank runs the
same workload on its own GPU (independent replicas, weak scaling, no
collective on the data path); the time is the max over ranks.

``--impl reference`` times the float64 CPU oracle on the host cores instead
(bounded row samples of the same workload), on rank 0 only.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s (and % of B200 dense BF16 peak) and ms/call at 1 GPU"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0  # B200 dense BF16 (the vendor's figure without sparsity), context only


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def captured_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu capture of this workload's
    kernel (a profiles/*.json record whose "workload" is this one), or None
    when there is none or the kernel's source files (the record's
    "source_files", by default fa_fwd_tc.cuh and ptx.cuh) have changed since
    the counters were taken."""
    import glob
    import hashlib

    csrc = os.path.join(ROOT, "tiled_attention_13_b200", "csrc")
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.json"))):
        rec = json.load(open(path))
        if rec.get("workload") != workload or "dram_bytes_per_launch" not in rec:
            continue
        files = rec.get("source_files", ["fa_fwd_tc.cuh", "ptx.cuh"])
        sha = hashlib.sha256(b"".join(open(os.path.join(csrc, f), "rb").read() for f in files)).hexdigest()
        if rec.get("kernel_source_sha256") == sha:
            return float(rec["dram_bytes_per_launch"])
    return None


def step_percentiles(ms):
    """p10 / median / p90 of per-step durations (nearest rank)."""
    xs = sorted(ms)
    pick = lambda q: xs[min(len(xs) - 1, max(0, int(round(q * (len(xs) - 1)))))]
    return {"p10": pick(0.1), "median": pick(0.5), "p90": pick(0.9)}


def roofline_bound(wl, peaks) -> str:
    """"tensor" when the workload's arithmetic intensity (algorithmic FLOPs
    per compulsory byte) reaches the measured ridge point, else "hbm"."""
    ridge = float(peaks["bf16_tflops"]) * 1e12 / (float(peaks["hbm_gbs"]) * 1e9)
    return "tensor" if wl.flops / wl.bytes_min >= ridge else "hbm"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.gpu), "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[5:]))
                except (ValueError, IndexError):
                    continue
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05]
        use = inside if inside else rows
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in use:
            for n, v in zip(names, r[3][1:5]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": sorted(reasons), "samples": len(use), "samples_in_timed_region": len(inside)}


# ------------------------------------------------------------------ CPU oracle baseline
def oracle_sample(wl, rows_budget_s: float = 12.0, seed: int = 0):
    """Time the float64 oracle (as it stands) on a bounded sample of ``wl``:
    whole query-row blocks of one head, until about ``rows_budget_s`` seconds of
    CPU work.  Returns (tflops, sample description, threads)."""
    import numpy as np
    import torch
    from threadpoolctl import threadpool_info

    from oracle import attention, attention_masked, band_mask, block_sparse_mask
    from tiled_attention_13_b200.inputs import make_block_mask, make_qkv

    one = wl.with_(B=1, H=1, Hkv=0)
    if wl.backward:  # the backward oracle on the first n positions of one head, repeated up to the budget
        from oracle import attention_backward
        from tiled_attention_13_b200.inputs import make_dout

        n = min(wl.Nq, wl.Nkv, 2048)
        small = one.with_(Nq=n, Nkv=n)
        q, k, v = make_qkv(small, device="cpu")
        do = make_dout(small, device="cpu")
        sl = (lambda t: t[0, :, 0]) if wl.layout == "BSND" else (lambda t: t[0, 0])
        q, k, v, do = (sl(t).to(torch.float64).numpy() for t in (q, k, v, do))
        flops, reps = 0.0, 0
        t0 = time.perf_counter()
        while True:
            attention_backward(q, k, v, do, causal=wl.causal)
            flops += small.flops
            reps += 1
            if time.perf_counter() - t0 > rows_budget_s:
                break
        el = time.perf_counter() - t0
        threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
        return flops / el / 1e12, (f"{reps} x the backward of the first {n} positions of one head of {wl.name}, "
                                   "float64 numpy oracle"), threads, el
    q, k, v = make_qkv(one, device="cpu")
    bmask = None
    if wl.block_density > 0:  # this head's block mask, expanded and cut to the causal range
        bmask = block_sparse_mask(make_block_mask(wl)[0, 0].numpy(), 128, 128, wl.Nq, wl.Nkv)
        if wl.causal:
            bmask &= np.tril(np.ones((wl.Nq, wl.Nkv), dtype=bool))
    if wl.layout == "BSND":
        q, k, v = q[0, :, 0], k[0, :, 0], v[0, :, 0]
    else:
        q, k, v = q[0, 0], k[0, 0], v[0, 0]
    qn, kn, vn = (t.to(torch.float64).numpy() for t in (q, k, v))
    block = 512
    flops = 0.0
    t0 = time.perf_counter()
    rows_done = 0
    # row blocks taken evenly over the sequence so causal work is representative;
    # when one head's rows take less than the budget (decoding: a row or a few),
    # the same head's data stands for the workload's next heads, up to B*H
    starts = list(range(0, wl.Nq, block))
    rng = np.random.default_rng(seed)
    rng.shuffle(starts)
    for r0 in [r for _ in range(wl.B * wl.H) for r in starts]:
        r1 = min(wl.Nq, r0 + block)
        if bmask is not None:
            mk = bmask[r0:r1]
            keep = mk.any(axis=1)
            attention_masked(qn[r0:r1][keep], kn, vn, mk[keep])
            flops += 4.0 * wl.d * float(mk.sum())
            rows_done += r1 - r0
            if time.perf_counter() - t0 > rows_budget_s:
                break
            continue
        if wl.band:
            mask = band_mask(wl.Nq, wl.Nkv, wl.band[0], wl.band[1])[r0:r1]
            attention_masked(qn[r0:r1], kn, vn, mask)
            flops += 4.0 * wl.d * float(mask.sum())
            rows_done += r1 - r0
            if time.perf_counter() - t0 > rows_budget_s:
                break
            continue
        attention(qn[r0:r1], kn, vn, causal=wl.causal, row_offset=r0)
        if wl.causal:
            flops += 4.0 * wl.d * sum(min(i + 1, wl.Nkv) for i in range(r0, r1))
        else:
            flops += 4.0 * wl.d * (r1 - r0) * wl.Nkv
        rows_done += r1 - r0
        if time.perf_counter() - t0 > rows_budget_s:
            break
    el = time.perf_counter() - t0
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    heads_done = -(-rows_done // wl.Nq)
    desc = (f"{rows_done} query rows (blocks of {block}) of one head of {wl.name}"
            + (f", its data standing for {heads_done} heads" if heads_done > 1 else "") + ", float64 numpy oracle")
    return flops / el / 1e12, desc, threads, el


# ------------------------------------------------------------------ main arms
def run_reference(args, wl):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import torch
    from threadpoolctl import threadpool_info

    torch.set_num_threads(len(os.sched_getaffinity(0)))
    per_step = []
    total_flops = 0.0
    desc = ""
    threads = 1
    for i in range(args.warmup + args.steps):
        tf, desc, threads, el = oracle_sample(wl, rows_budget_s=args.ref_step_s, seed=i)
        if i >= args.warmup:
            per_step.append(el)
            total_flops += tf * el * 1e12
    el = sum(per_step)
    value = total_flops / el / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * el / max(1, len(per_step)), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(wl, ws),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": "each step: " + desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


L2_BYTES = 126 * 2**20


def n_input_sets(wl) -> int:
    """Input sets to rotate: >= 2, and >= 2x the L2 size in total."""
    return max(2, -(-2 * L2_BYTES // int(wl.bytes_min)))


def _config(wl, ws):
    n = n_input_sets(wl)
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "Nq": wl.Nq, "Nkv": wl.Nkv, "d": wl.d,
            "layout": wl.layout, "causal": wl.causal, "input_dtype": wl.dtype,
            **({"Hkv": wl.kv_heads} if wl.kv_heads != wl.H else {}),
            **({"kv_cache": f"paged, {wl.block_size}-key blocks in shuffled order"} if wl.block_size > 0 else {}),
            **({"band": {"pre_tokens": wl.band[0], "next_tokens": wl.band[1]}} if wl.band else {}),
            **({"num_splits": wl.num_splits} if wl.num_splits >= 0 else {}),
            **({"block_sparse": f"128x128 blocks, density {wl.block_density} per head plus the diagonal"
                + (", intersected with the causal mask" if wl.causal else "")} if wl.block_density > 0 else {}),
            "parallelism": f"independent replicas x{ws} (no collective)",
            "l2": (f"{n} input sets of {wl.bytes_min / 1e6:.1f} MB (Q, K, V, O, LSE) rotate between steps, "
                   f"{n * wl.bytes_min / 1e6:.0f} MB in all > 2x the 126 MB L2"),
            "flops_per_step_per_gpu": wl.flops}


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    import tiled_attention_13_b200 as fa
    from tiled_attention_13_b200.inputs import make_qkv

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    fa.lib()
    stream = torch.cuda.current_stream(dev)

    sets = []
    n_sets = n_input_sets(wl)
    for s in range(n_sets):
        q, k, v = make_qkv(wl.with_(seed=wl.seed + s), device=dev)
        o = torch.empty_like(q)
        lse = torch.empty((wl.B, wl.H, wl.Nq), dtype=torch.float32, device=dev)
        paged = None
        if wl.block_size > 0:  # K/V through a paged cache built from the same keys and values
            from tiled_attention_13_b200.inputs import make_paged_kv

            paged = make_paged_kv(wl.with_(seed=wl.seed + s), k, v)
        sets.append((q, k, v, o, lse, paged))
    bmask = None
    if wl.block_density > 0:
        from tiled_attention_13_b200.inputs import make_block_mask

        bmask = make_block_mask(wl, device=dev)
    bwd = []  # backward: per input set the forward's O and LSE, dO, the gradients and the workspace
    if wl.backward:
        from tiled_attention_13_b200.inputs import make_dout

        _, nbytes = fa.fa_bwd_workspace_size(wl.B, wl.H, wl.Nq, wl.d)
        for s_i, (q, k, v, o, lse, _) in enumerate(sets):
            fa.forward(q, k, v, causal=wl.causal, layout=wl.layout, out=o, lse=lse)
            bwd.append((make_dout(wl.with_(seed=wl.seed + s_i), device=dev), torch.empty_like(q), torch.empty_like(k),
                        torch.empty_like(v), torch.empty(nbytes, dtype=torch.uint8, device=dev)))
    torch.cuda.synchronize()

    splits = wl.num_splits if wl.num_splits >= 0 else None
    # kernels per step: the split kernel and the merge when the plan has
    # more than one slice, else the one attention kernel
    launches_per_step, s_used = 1, None
    if wl.backward:
        launches_per_step = 3  # row statistics, the gradient kernel, dQ conversion (plus one memset)
    if splits is not None:
        s_used, _ = fa.splitkv_plan(wl.B, wl.H, wl.Nq, wl.Nkv, wl.d, splits)
        launches_per_step = 2 if s_used > 1 else 1

    def step(i):
        q, k, v, o, lse, paged = sets[i % n_sets]
        if wl.backward:
            do, dq, dk, dv, ws = bwd[i % n_sets]
            rc = fa.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                           dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws.numel(), wl.B, wl.H,
                           wl.kv_heads, wl.Nq, wl.Nkv, wl.d, -1.0, int(wl.causal),
                           fa.FA_LAYOUT_BHND if wl.layout == "BHND" else fa.FA_LAYOUT_BSND, fa.FA_DTYPE_BF16,
                           torch.cuda.current_stream().cuda_stream)
            if rc != 0:
                raise RuntimeError(f"fa_bwd: {fa.fa_status_string(rc)}")
            return
        if paged is None:
            fa.forward(q, k, v, causal=wl.causal, layout=wl.layout, out=o, lse=lse, band=wl.band or None,
                       num_splits=splits, block_mask=bmask)
        else:
            kc, vc, table = paged
            fa.forward_paged(q, kc, vc, table, wl.Nkv, causal=wl.causal, layout=wl.layout, out=o, lse=lse,
                             num_splits=splits)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    rc = fa.fa_get_device_status(stream.cuda_stream)
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {fa.fa_status_string(rc)}")

    sampler = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local])
                           if "CUDA_VISIBLE_DEVICES" in os.environ else local)
    if rank == 0:
        sampler.start()
        time.sleep(0.3)
    # The K timed steps are recorded once into a CUDA graph (with an event
    # pair around every launch) and replayed: the device then runs the steps
    # back to back and host launch overhead stays out of the timing, which
    # matters for calls of a few microseconds.  --no-graph launches eagerly.
    # Two graphs of the same K steps: the timed one has no nodes but the
    # kernels (event records between microsecond-scale kernels cost time of
    # their own); the second, replayed after the timed region, records an
    # event pair around every step for the per-kernel times.
    use_graph = not args.no_graph
    ev = [(torch.cuda.Event(enable_timing=True, external=use_graph),
           torch.cuda.Event(enable_timing=True, external=use_graph)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    graph = graph_ev = None
    if use_graph:
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        graph, graph_ev = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.stream(cap):
            graph.capture_begin()
            for i in range(args.steps):
                step(i)
            graph.capture_end()
            graph_ev.capture_begin()
            for i in range(args.steps):
                ev[i][0].record(cap)
                step(i)
                ev[i][1].record(cap)
            graph_ev.capture_end()
        stream.wait_stream(cap)
        graph.replay()  # untimed: uploads the graphs
        graph_ev.replay()
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    start.record(stream)
    if use_graph:
        graph.replay()
    else:
        for i in range(args.steps):
            ev[i][0].record(stream)
            step(i)
            ev[i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    if ws > 1:
        dist.barrier()
    total_ms = start.elapsed_time(end)
    if use_graph:
        graph_ev.replay()  # the per-step event pairs, after the timed region
        torch.cuda.synchronize()
    kern_ms = [a.elapsed_time(b) for a, b in ev]
    if rank == 0:
        time.sleep(0.1)
        sampler.stop()
    rc = fa.fa_get_device_status(stream.cuda_stream)
    if rc != 0:
        raise RuntimeError(f"device status after timing: {fa.fa_status_string(rc)}")

    # ---- steady state: the same K steps replayed back to back for about
    # --sustain-s seconds after the timed region, once the 1 kW power cap has
    # had time to act; reported beside (not in place of) the burst figure
    sustained = None
    if args.sustain_s > 0 and use_graph:
        reps = max(1, int(args.sustain_s * 1e3 / max(total_ms, 1e-3)))
        ssamp = ClockSampler(sampler.gpu)
        if rank == 0:
            ssamp.start()
            time.sleep(0.3)
        a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if ws > 1:
            dist.barrier()
        ts0 = time.time()
        a_ev.record(stream)
        for _ in range(reps):
            graph.replay()
        b_ev.record(stream)
        torch.cuda.synchronize()
        ts1 = time.time()
        if rank == 0:
            time.sleep(0.1)
            ssamp.stop()
        rc = fa.fa_get_device_status(stream.cuda_stream)
        if rc != 0:
            raise RuntimeError(f"device status after the steady-state run: {fa.fa_status_string(rc)}")
        ms_s = max_over_ranks(a_ev.elapsed_time(b_ev), dev) / (reps * args.steps)
        sustained = {"seconds": reps * args.steps * ms_s / 1e3, "steps": reps * args.steps, "ms_per_step": ms_s,
                     "value": ws * wl.flops / (ms_s * 1e-3) / 1e12, "unit": UNIT,
                     "clocks": ssamp.summary(ts0, ts1) if rank == 0 else None}

    ms_step = max_over_ranks(total_ms, dev) / args.steps
    value = ws * wl.flops / (ms_step * 1e-3) / 1e12

    # ---- end-to-end through the public API: pinned host in, host out
    e2e = None
    if not args.no_e2e and (wl.block_size > 0 or wl.band or splits is not None or bmask is not None or wl.backward):
        e2e = {"value": None, "unit": UNIT, "skipped": "HostPipeline runs the plain forward (contiguous K/V, no band, "
               "block mask or split-KV); this path is measured on the device only"}
    elif not args.no_e2e:
        # Every step copies its inputs from pinned host memory and reads its
        # O and LSE back; HostPipeline overlaps step i+1's upload and step
        # i-1's download with step i's kernel (separate streams, two device
        # buffer sets).  Timed from the first upload to the last download.
        qh, kh, vh = (x.cpu().pin_memory() for x in sets[0][:3])
        oh = torch.empty_like(qh).pin_memory()
        lh = torch.empty((wl.B, wl.H, wl.Nq), dtype=torch.float32).pin_memory()
        hp = fa.HostPipeline(qh, kh, causal=wl.causal, layout=wl.layout, device=dev)
        for _ in range(3):
            hp.submit(qh, kh, vh, oh, lh)
        hp.synchronize()
        n_e2e = max(3, min(args.steps, 20))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if ws > 1:
            dist.barrier()
        a.record(hp.up)
        for _ in range(n_e2e):
            hp.submit(qh, kh, vh, oh, lh)
        b.record(hp.down)
        hp.synchronize()
        te = max_over_ranks(a.elapsed_time(b) / n_e2e, dev)
        e2e = {"value": ws * wl.flops / (te * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": hp.h2d_bytes, "d2h_bytes_per_step": hp.d2h_bytes,
               "ms_per_step": te, "steps": n_e2e,
               "form": "HostPipeline: upload, kernel and download of neighbouring steps overlap"}
        del hp, qh, kh, vh, oh, lh

    if rank == 0:
        peaks, src = load_peaks()
        # a step's kernel time is at most its event-pair time and at most the
        # timed graph's time per step (kernel plus the gap to the next)
        kmean = min(sum(kern_ms) / len(kern_ms), ms_step)
        traffic = args.traffic if args.traffic is not None else captured_traffic(wl.name)
        achieved = wl.flops / (kmean * 1e-3) / 1e12
        bound = roofline_bound(wl, peaks)
        if bound == "tensor":
            peak = float(peaks["bf16_tflops"])
            roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": traffic,
                    "peak_source": f"{src} bf16_tflops (burst; sustained {peaks.get('bf16_tflops_sustained')})",
                    "kernel_ms_mean": kmean, "event_pair_ms_min": min(kern_ms)}
        else:
            gbs = wl.bytes_min / (kmean * 1e-3) / 1e9
            peak = float(peaks["hbm_gbs"])
            roof = {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                    "traffic": traffic, "peak_source": f"{src} hbm_gbs", "kernel_ms_mean": kmean,
                    "event_pair_ms_min": min(kern_ms), "algorithmic_bytes": wl.bytes_min}
        if sustained is not None:
            if bound == "tensor":
                sp = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
                sustained.update({"peak": sp, "peak_source": f"{src} bf16_tflops_sustained",
                                  "frac": (sustained["value"] / ws) / sp})
            else:
                gbs = wl.bytes_min / (sustained["ms_per_step"] * 1e-3) / 1e9
                sustained.update({"achieved_gbs": gbs, "peak": float(peaks["hbm_gbs"]),
                                  "peak_source": f"{src} hbm_gbs", "frac": gbs / float(peaks["hbm_gbs"])})
        if launches_per_step > 1 and wl.backward:
            roof["timed"] = ("each step's event pair spans the accumulator clear and the three backward kernels; "
                             "achieved counts the backward's algorithmic FLOPs (2.5x the forward's)")
        elif launches_per_step > 1:
            roof["timed"] = ("each step's event pair spans both kernels (split kernel and merge); achieved "
                             "counts the compulsory bytes only")
        cpu = None
        if not args.no_cpu_baseline and ws == 1:
            tf, desc, threads, el = oracle_sample(wl, rows_budget_s=args.cpu_budget_s)
            cpu = {"value": tf, "unit": UNIT, "cores": threads, "kind": "oracle",
                   "sample": desc + f" ({el:.1f} s)"}
        clocks = sampler.summary(t0, t1)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else wl.dtype,
            "data": "synthetic: seeded i.i.d. N(0,1) Q/K/V of the workload's shape",
            "config": _config(wl, ws), "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * launches_per_step, "clocks": clocks,
            "timing": ("cuda-graph replay of the K steps (kernel nodes only); per-step times from a second replay "
                       "with an event pair around each step") if use_graph else "eager launches",
            "pct_of_measured_bf16_peak": 100.0 * (value / ws) / float(peaks["bf16_tflops"]),
            "pct_of_datasheet_bf16_peak": 100.0 * (value / ws) / DATASHEET_BF16_TFLOPS,
            "event_pair_ms_percentiles": step_percentiles(kern_ms),
            "steady_state": sustained,
        }
        if s_used is not None:
            line["config"]["splits_used"] = s_used
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama13b-8k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--num-splits", type=int, default=None,
                    help="override the workload's split-KV setting: -1 unsplit, 0 the library's count, n slices")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the timed steps eagerly instead of as one CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--ref-step-s", type=float, default=2.0)
    ap.add_argument("--sustain-s", type=float, default=1.0,
                    help="after the timed region, replay the timed steps for about this many seconds and report "
                         "the steady-state figure beside the burst one (0: skip)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch from an ncu capture of the same kernel (else null)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from tiled_attention_13_b200.inputs import WORKLOADS

    wl = WORKLOADS[args.workload]
    if args.num_splits is not None:
        wl = wl.with_(num_splits=args.num_splits)
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
