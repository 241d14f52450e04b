"""Benchmark: DS4 sparse-prefill tokens/s on the 10,240-token frontier workload.

One step = one whole prefill of T = 10,240 tokens: five 2,048-token bands in
chronological order, each running indexer -> top-k -> streaming sparse MLA
attention through the C ABI (ds4sp_prefill_band). Inputs are seeded synthetic
tensors resident in HBM before the timed region; per step the inputs read
(q 189 MB, q_idx 168 MB) and the output written (335 MB) exceed the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]

N > 1 runs under torchrun: each rank prefills its own sequence (weak scaling, no
collective on the data path); timing is the max over ranks. ``--impl reference``
times the CPU oracle (the only reference this method has) on a bounded token
sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_mla_prefill_b200 import ds4sp as D  # noqa: E402
from sparse_mla_prefill_b200.inputs import generate, workload  # noqa: E402

WORKLOAD = "10k"
METRIC = "sparse-prefill attention tokens/s at 8K/10K; HBM GB/s and % of roofline"


# ------------------------------------------------------------------ algorithmic work

def n_vis(t, ratio=4):
    return (t + 1) // ratio


def attn_rows(T, k, n_swa, t0=0, t1=None):
    t1 = T if t1 is None else t1
    return sum(min(k, n_vis(t)) + min(n_swa, t + 1) for t in range(t0, t1))


def algorithmic(wl):
    """Per-step algorithmic bytes / FLOPs of each kernel: attention 1152 B per (token,
    attended row) plus Q, O and index bytes per token; indexer 2*H_i*D_i FLOPs per (token,
    visible row); top-k 4 B per (token, visible row) read plus 4*k B per token written."""
    T, k, n_swa = wl.T, wl.top_k, wl.n_swa
    rows = attn_rows(T, k, n_swa)
    sum_vis = sum(n_vis(t) for t in range(T))
    return {
        "attention_bytes": 1152 * rows + (18432 + 32768 + 4 * k) * T,
        "attention_flops": 2 * 16 * (576 + 512) * rows,
        "indexer_flops": 2 * wl.H_i * wl.D_i * sum_vis,
        "indexer_bytes": 2 * wl.H_i * wl.D_i * T + 4 * wl.H_i * T + 4 * sum_vis,
        "topk_bytes": 4 * sum_vis + 4 * k * T,
        "rows": rows,
    }


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def attention_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, or None when the
    kernel's sources changed after that capture (the figure would no longer apply)."""
    import hashlib
    import re
    prof = os.path.join(ROOT, "profiles", "sparse_attn_mma_kernel_10k_band4.md")
    csrc = os.path.join(ROOT, "sparse_mla_prefill_b200", "csrc")
    try:
        text = open(prof).read()
        src = b"".join(open(os.path.join(csrc, f), "rb").read()
                       for f in ("sparse_attn_mma.cuh", "device_common.cuh"))
    except OSError:
        return None
    want = re.search(r"kernel_source_sha256: ([0-9a-f]+)", text)
    val = re.search(r"traffic_bytes_per_launch: ([0-9]+)", text)
    if not want or not val or hashlib.sha256(src).hexdigest()[:16] != want.group(1):
        return None
    return int(val.group(1))


# ------------------------------------------------------------------ ranks

def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value (every rank takes part in the same all-reduce)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_throughput(tokens_per_rank: int, world: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms_max / 1e3)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in out.splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ reference arm (oracle)

def blas_threads():
    """Threads NumPy's BLAS runs the oracle's matrix products on."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return torch.get_num_threads()


def cpu_oracle_sample(wl, n_sample, inputs_np=None, return_result=False, one_core=False):
    """Time the float64 CPU oracle on a spread sample of tokens; tokens/s (and, with
    return_result, the oracle's indices and outputs for those tokens). one_core limits
    NumPy's BLAS to one thread for the timing."""
    import contextlib
    import oracle
    if inputs_np is None:
        inputs_np = {k: v.numpy() for k, v in generate(wl).items()}
    stride = max(1, wl.T // n_sample)
    toks = list(range(stride - 1, wl.T, stride))[:n_sample]
    ctx = contextlib.nullcontext()
    if one_core:
        from threadpoolctl import threadpool_limits
        ctx = threadpool_limits(limits=1)
    with ctx:
        cores = 1 if one_core else blas_threads()
        t0 = time.perf_counter()
        ref = oracle.prefill_tokens(inputs_np, toks, wl.top_k, wl.n_swa)
        dt = time.perf_counter() - t0
    line = {"value": len(toks) / dt, "unit": "tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{len(toks)} of {wl.T} tokens (every {stride}th), float64 NumPy, "
                      f"{dt:.1f} s"}
    return (line, ref) if return_result else line


def sampled_parity(ref, topk_gpu, out_gpu, of="ds4sp_prefill_host result (pinned host buffers)"):
    """The end-to-end result against the oracle on its sampled tokens: indices bit for
    bit, attention max-abs and NMSE over every element of those tokens."""
    import numpy as np
    toks = ref["tokens"]
    got = out_gpu[toks].astype(np.float64)
    err = got - ref["out"]
    max_abs = float(np.abs(err).max())
    nmse = float((err ** 2).sum() / (ref["out"] ** 2).sum())
    exact = bool(np.array_equal(topk_gpu[toks], ref["topk"]))
    return {"tokens": int(len(toks)), "topk_bit_exact": exact, "max_abs": max_abs, "nmse": nmse,
            "bar": {"max_abs": 2e-3, "nmse": 1e-6},
            "pass": exact and max_abs <= 2e-3 and nmse <= 1e-6, "of": of}


def run_reference(args, rank, world):
    wl = workload(WORKLOAD)
    if rank != 0:
        return
    inputs_np = {k: v.numpy() for k, v in generate(wl).items()}
    # a bounded sample per step, so that the whole run stays within a few minutes
    per_step = max(8, min(256, 8192 // max(1, args.steps)))
    for _ in range(args.warmup):
        cpu_oracle_sample(wl, 32, inputs_np)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(cpu_oracle_sample(wl, per_step, inputs_np))
    wall = time.perf_counter() - t0
    value = args.steps * per_step / wall
    cb = dict(vals[-1])
    cb["value"] = value
    cb["sample"] = f"{args.steps} steps x {per_step} tokens spread over the {wl.T}-token sequence"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * wall / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": config_name(wl), "sample_tokens_per_step": per_step},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def config_name(wl):
    return (f"{wl.name}: T={wl.T} as {wl.n_bands} bands of {wl.band}, 16 heads, d_qk 576 / d_v 512 "
            f"fp16, indexer {wl.H_i}x{wl.D_i}, top_k {wl.top_k}, n_swa {wl.n_swa}, seed {wl.seed}")


# ------------------------------------------------------------------ our arm

def verify_latency(dev, reps: int = 50):
    """Latency of one verify step per width q: ds4sp_indexer_topk + ds4sp_sparse_attn on
    the last q tokens of the 122,880-token verify workload (q = 1..5), device-resident
    inputs, CUDA events around `reps` back-to-back steps."""
    wl = workload("verify")
    d = {k: v.to(dev) for k, v in generate(wl).items()}
    T = wl.T
    cfg = D.make_config(n_idx_heads=wl.H_i, d_idx=wl.D_i, top_k=wl.top_k, n_swa=wl.n_swa,
                        max_tokens=T, band=wl.band)
    h = D.ds4sp_create(cfg)
    res = {}
    try:
        for q in range(1, 6):
            sl = {k: (v[5 - q:].contiguous() if k in ("q", "q_idx", "w") else v) for k, v in d.items()}
            topk = torch.empty((q, wl.top_k), dtype=torch.int32, device=dev)
            out = torch.empty((q, 16, 512), dtype=torch.float32, device=dev)
            ws = torch.empty(max(D.ds4sp_workspace_bytes(h, T - q, q), 256), dtype=torch.uint8,
                             device=dev)

            def call():
                D.ds4sp_indexer_topk(h, sl["q_idx"], sl["k_idx"], sl["w"], T - q, q, topk, ws)
                D.ds4sp_sparse_attn(h, sl["q"], sl["kv_raw"], sl["kv_cmp"], topk, T - q, q, out)

            for _ in range(5):
                call()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                call()
            e1.record()
            torch.cuda.synchronize()
            res[f"q{q}"] = round(e0.elapsed_time(e1) / reps * 1e3, 1)
            # The same step captured once into a CUDA graph and replayed: the launches'
            # host cost (argument checks, schedules, three to four launches) leaves the
            # step's latency.
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                call()
            for _ in range(5):
                g.replay()
            torch.cuda.synchronize()
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            res[f"graph_q{q}"] = round(e0.elapsed_time(e1) / reps * 1e3, 1)
            del g
        st, bits = D.ds4sp_device_status(h)
        if st != D.OK:
            raise RuntimeError(f"device status {bits:#x} after verify timing")
    finally:
        D.ds4sp_destroy(h)
    return {"workload": "verify: 122,880-token context, the last q = 1..5 tokens, top_k 512, "
                        "n_swa 128, indexer 64x128, seed 4",
            "unit": "us per step (indexer + top-k + attention); q<n>: launched from the host "
                    "each step, graph_q<n>: one captured CUDA graph replayed", **res}


def config_throughput(name, dev, steps, stream):
    """tokens/s of one prefill workload (device-resident inputs, `steps` whole prefills
    between CUDA events on the launching stream); returns the line and the last result."""
    wl = workload(name)
    host = generate(wl)
    inputs = {k: v.to(dev) for k, v in host.items()}
    cfg = D.make_config(n_idx_heads=wl.H_i, d_idx=wl.D_i, top_k=wl.top_k, n_swa=wl.n_swa,
                        max_tokens=wl.T, band=wl.band)
    h = D.ds4sp_create(cfg)
    try:
        topk = torch.empty((wl.T, wl.top_k), dtype=torch.int32, device=dev)
        out = torch.empty((wl.T, 16, 512), dtype=torch.float32, device=dev)
        ws = D.band_workspace(h, wl.T, dev)
        for _ in range(3):
            D.prefill(h, inputs, wl.T, topk, out, ws, stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            D.prefill(h, inputs, wl.T, topk, out, ws, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        st, bits = D.ds4sp_device_status(h)
        if st != D.OK:
            raise RuntimeError(f"device status {bits:#x} after {name} timing")
        line = {"workload": config_name(wl), "tokens_per_s": wl.T * steps / (ms / 1e3),
                "ms_per_prefill": ms / steps, "steps": steps}
        return line, host, topk.cpu().numpy(), out.cpu().numpy()
    finally:
        D.ds4sp_destroy(h)


def gather_ceiling(dev, stream, rows_table=12800, n=6_020_672, reps=5):
    """Bandwidth of random 1152-byte row gathers from an L2-resident table of the 10K
    prefill's size (its 10,240 raw + 2,560 compressed rows, 14.75 MB), through the
    library's gather probe: the ceiling for the attention kernel's row traffic."""
    g = torch.Generator(device="cpu").manual_seed(5)
    table = torch.randn(rows_table, 576, generator=g).half().to(dev)
    idx = torch.randint(0, rows_table, (n,), generator=g, dtype=torch.int32).to(dev)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    props = torch.cuda.get_device_properties(dev)
    grid = props.multi_processor_count * 4
    for _ in range(3):
        D.ds4sp_probe_gather(table, idx, sink, grid, stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        D.ds4sp_probe_gather(table, idx, sink, grid, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    return {"GBps": 1152 * n / (ms / 1e3) / 1e9, "rows": n, "table_MB": rows_table * 1152 / 1e6,
            "ms": ms, "how": "ds4sp_probe_gather: random rows, 16-byte loads into registers, "
                             f"{grid} CTAs x 512 threads"}


def run_ours(args, rank, world, local_rank):
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = workload(WORKLOAD)
    alg = algorithmic(wl)
    pk = peaks()
    solo = rank == 0 and world == 1          # extras that only a single-GPU run reports

    host = generate(wl)
    inputs = {k: v.to(dev) for k, v in host.items()}
    cfg = D.make_config(n_idx_heads=wl.H_i, d_idx=wl.D_i, top_k=wl.top_k, n_swa=wl.n_swa,
                        max_tokens=wl.T, band=wl.band, topk_mode=args.topk_mode,
                        kv_format=args.kv_format, attn_kernel=args.attn_kernel)
    h = D.ds4sp_create(cfg)
    if args.kv_format:
        # a quantized cache of the same rows, made on the device before any timing
        for kv in ("kv_raw", "kv_cmp"):
            inputs[kv] = D.ds4sp_quantize_kv(inputs[kv], args.kv_format)
    # the tensors the end-to-end pass copies in (the quantized cache, if any)
    host_io = dict(host, kv_raw=inputs["kv_raw"].cpu(), kv_cmp=inputs["kv_cmp"].cpu())
    topk = torch.empty((wl.T, wl.top_k), dtype=torch.int32, device=dev)
    out = torch.empty((wl.T, 16, 512), dtype=torch.float32, device=dev)
    ws = D.band_workspace(h, wl.T, dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        D.prefill(h, inputs, wl.T, topk, out, ws, stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, bits = D.ds4sp_device_status(h)
    if st != D.OK:
        raise RuntimeError(f"device status {bits:#x} after warm-up")

    def timed_steps(n):
        barrier()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(n):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return ev0.elapsed_time(ev1)

    clocks = ClockSampler(local_rank)
    clocks.start()
    # `value`: K steps with nothing but the steps in the stream. The library's events
    # around each kernel put a timestamp between every two launches, which by itself
    # lengthens a prefill by about 6% (1.39 -> 1.47 ms at 10K on B200), so the per-kernel
    # split and the roofline come from a second pass of the same K steps with them on.
    ms = timed_steps(args.steps)
    D.ds4sp_profile_enable(h, True)
    D.ds4sp_profile_read(h)
    ms_prof = timed_steps(args.steps)
    prof = D.ds4sp_profile_read(h)
    D.ds4sp_profile_enable(h, False)
    # The K timed steps last tens of milliseconds, shorter than the sampler's 100 ms
    # period; the same step keeps running for about `soak` seconds more so that the clock
    # record holds enough samples under this load.
    soak_steps = max(1, int(args.soak * 1e3 / max(ms / args.steps, 1e-3)))
    ms_soak = timed_steps(soak_steps)
    clk = clocks.stop()
    clk["window"] = (f"sampled every 100 ms over the timed steps, the profiled pass and "
                     f"{soak_steps} more steps ({ms_soak / 1e3:.2f} s) of the same prefill")
    ms_max = max_over_ranks(ms, world, dev)
    ms_prof_max = max_over_ranks(ms_prof, world, dev)
    # The fused step has no separate indexer and top-k launches: their own figures come
    # from the same steps in the two-kernel form (topk_mode 0), timed the same way.
    split = None
    if args.topk_mode == 1:
        cfg2 = D.make_config(n_idx_heads=wl.H_i, d_idx=wl.D_i, top_k=wl.top_k, n_swa=wl.n_swa,
                             max_tokens=wl.T, band=wl.band, topk_mode=0,
                             kv_format=args.kv_format, attn_kernel=args.attn_kernel)
        h2 = D.ds4sp_create(cfg2)
        try:
            for _ in range(3):
                D.prefill(h2, inputs, wl.T, topk, out, ws, stream)
            torch.cuda.synchronize()
            D.ds4sp_profile_enable(h2, True)
            D.ds4sp_profile_read(h2)
            for _ in range(args.steps):
                D.prefill(h2, inputs, wl.T, topk, out, ws, stream)
            torch.cuda.synchronize()
            split = D.ds4sp_profile_read(h2)
            st, bits = D.ds4sp_device_status(h2)
            if st != D.OK:
                raise RuntimeError(f"device status {bits:#x} in the two-kernel pass")
        finally:
            D.ds4sp_destroy(h2)

    # end to end through the public API: pinned host inputs -> device, prefill, out -> host
    pinned = {k: v.pin_memory() for k, v in host_io.items()}
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = out.numel() * out.element_size()
    e2e_steps = max(1, min(args.steps, 5))
    D.prefill_host(h, pinned, inputs, wl.T, topk, out, ws, out_host, stream)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        D.prefill_host(h, pinned, inputs, wl.T, topk, out, ws, out_host, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    st, bits = D.ds4sp_device_status(h)
    if st != D.OK:
        raise RuntimeError(f"device status {bits:#x} after timing")
    # The end-to-end result, kept for the parity check against the oracle's sample below
    # (the variants after this overwrite the device buffers).
    out_e2e = out_host.numpy().copy()
    topk_e2e = topk.cpu().numpy()

    verify = None
    if solo and not args.no_verify:
        verify = verify_latency(dev)

    # The same step with other configuration choices (VARIANTS below: ex2.approx instead
    # of exp2f, fp32-staged probabilities in P . V, the two-kernel top-k, quantized
    # caches, ...), for comparison; not the headline.
    variants = None
    if solo and not args.no_verify:
        variants = {}
        for name, modes in VARIANTS:
            cfg_v = D.make_config(n_idx_heads=wl.H_i, d_idx=wl.D_i, top_k=wl.top_k,
                                  n_swa=wl.n_swa, max_tokens=wl.T, band=wl.band, **modes)
            hv = D.ds4sp_create(cfg_v)
            inp_v = inputs
            if modes.get("kv_format"):
                # the same cache, quantized on the device (outside the timed region)
                inp_v = dict(inputs)
                for kv in ("kv_raw", "kv_cmp"):
                    inp_v[kv] = D.ds4sp_quantize_kv(inputs[kv], modes["kv_format"], stream=stream)
            try:
                for _ in range(3):
                    D.prefill(hv, inp_v, wl.T, topk, out, ws, stream)
                torch.cuda.synchronize()
                n_var = 20
                ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                ev0.record(stream)
                for _ in range(n_var):
                    D.prefill(hv, inp_v, wl.T, topk, out, ws, stream)
                ev1.record(stream)
                torch.cuda.synchronize()
                D.ds4sp_profile_enable(hv, True)
                D.ds4sp_profile_read(hv)
                for _ in range(n_var):
                    D.prefill(hv, inp_v, wl.T, topk, out, ws, stream)
                torch.cuda.synchronize()
                vprof = D.ds4sp_profile_read(hv)
                st, bits = D.ds4sp_device_status(hv)
                if st != D.OK:
                    raise RuntimeError(f"device status {bits:#x} in variant {name}")
                variants[name] = {"ms_per_step": ev0.elapsed_time(ev1) / n_var,
                                  **{f"{k}_ms_per_step": v[0] / n_var for k, v in vprof.items()},
                                  "steps": n_var, **modes}
            finally:
                D.ds4sp_destroy(hv)

    # tokens/s of every prefill workload (the 10K line is the headline; the others use the
    # same step on their own sizes), and all-token parity of the 8K prefill.
    per_config = parity_8k = None
    if solo and not args.no_per_config:
        per_config = {}
        for name in ("band", "8k"):
            line_c, host_c, tk_c, out_c = config_throughput(name, dev, max(args.steps, 20), stream)
            per_config[name] = line_c
            if name == "8k" and not args.no_cpu_baseline:
                wl8 = workload("8k")
                ref8 = cpu_oracle_sample(wl8, wl8.T, {k: v.numpy() for k, v in host_c.items()},
                                         return_result=True)[1]
                parity_8k = sampled_parity(ref8, tk_c, out_c,
                                           of="every token of the 8,192-token prefill "
                                              "(ds4sp_prefill_band, device buffers)")
        per_config["10k"] = {"workload": config_name(wl), "tokens_per_s": wl.T * args.steps / (ms / 1e3),
                             "ms_per_prefill": ms / args.steps, "steps": args.steps}

    l2 = None
    if solo:
        l2 = gather_ceiling(dev, stream)

    cpu_base = parity = None
    if solo and not args.no_cpu_baseline and not args.kv_format:
        cpu_base, ref = cpu_oracle_sample(wl, args.cpu_sample,
                                          {k: v.numpy() for k, v in host.items()},
                                          return_result=True)
        one = cpu_oracle_sample(wl, 256, {k: v.numpy() for k, v in host.items()}, one_core=True)
        cpu_base["one_core"] = {"value": one["value"], "cores": 1, "sample": one["sample"]}
        parity = sampled_parity(ref, topk_e2e, out_e2e)

    if rank == 0:
        value = job_throughput(wl.T, world, args.steps, ms_max)
        attn_ms, attn_n = prof["attention"]
        head_launches = attn_n + prof["indexer"][1] + prof["topk"][1]
        fused = None
        # (a headline step with separate top-k launches did not take the fused kernel)
        if split is not None and prof["topk"][1] == 0:
            f_ms, f_n = prof["indexer"]           # the fused kernel's launches
            f_tf = alg["indexer_flops"] * args.steps / (f_ms / 1e3) / 1e12
            fused = {"ms_per_step": f_ms / args.steps, "launches": f_n,
                     "indexer_TFLOPs": f_tf, "frac_tensor_indexer_flops": f_tf / pk["bf16_tflops"],
                     "how": "indexer + top-k in one kernel, the headline step's; the "
                            "indexer and top-k figures come from the two-kernel pass"}
            idx_ms, idx_n = split["indexer"]
            topk_ms, topk_n = split["topk"]
        else:
            idx_ms, idx_n = prof["indexer"]
            topk_ms, topk_n = prof["topk"]
        steps = args.steps
        attn_achieved = alg["attention_bytes"] * steps / (attn_ms / 1e3) / 1e9
        idx_achieved = alg["indexer_flops"] * steps / (idx_ms / 1e3) / 1e12
        attn_kernel = {"ms_per_step": attn_ms / steps, "launches": attn_n,
                       "alg_GBps": attn_achieved,
                       "frac_hbm": attn_achieved / pk["hbm_gbs"],
                       "alg_bytes_per_step": alg["attention_bytes"]}
        if l2:
            # the rows and Q the kernel reads through L2, against the measured gather ceiling
            l2_bytes = 1152 * alg["rows"] + 18432 * wl.T
            l2_gbs = l2_bytes * steps / (attn_ms / 1e3) / 1e9
            attn_kernel["l2_GBps"] = l2_gbs
            attn_kernel["frac_l2_gather"] = l2_gbs / l2["GBps"]
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": ms_max / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16", "data": "synthetic",
            "config": {"workload": config_name(wl), "parallelism": f"dp{world} (one sequence per rank)",
                       "l2": "inputs larger than L2: q+q_idx read and out written per step = 692 MB > 126 MB"},
            "roofline": {"bound": "hbm", "achieved": attn_achieved, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": attn_achieved / pk["hbm_gbs"],
                         "traffic": attention_traffic(), "kernel": "sparse_attn_mma_kernel",
                         "peak_source": f"{pk['source']} hbm_gbs (of {pk['source']})",
                         "l2_gather_frac": attn_kernel.get("frac_l2_gather")},
            "kernels": {
                "attention": attn_kernel,
                "indexer": {"ms_per_step": idx_ms / steps, "launches": idx_n,
                            "TFLOPs": idx_achieved,
                            "frac_tensor": idx_achieved / pk["bf16_tflops"],
                            "alg_flops_per_step": alg["indexer_flops"],
                            "from": "two-kernel pass (topk_mode 0)" if fused else "headline pass"},
                "topk": {"ms_per_step": topk_ms / steps, "launches": topk_n,
                         "alg_GBps": (alg["topk_bytes"] * steps / (topk_ms / 1e3) / 1e9
                                      if topk_ms > 0 else None),
                         "from": "two-kernel pass (topk_mode 0)" if fused else "headline pass"},
                "indexer_topk_fused": fused,
            },
            "gpu_launches": head_launches,
            "kernel_timing": {"steps": steps, "ms_per_step": ms_prof_max / steps,
                              "how": "a second pass of the same steps with CUDA events "
                                     "around each kernel on the launching stream"},
            "per_config": per_config,
            "l2_gather_ceiling": l2,
            "verify": verify,
            "variants": variants,
            "e2e": {"value": job_throughput(wl.T, world, e2e_steps, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "clocks": clk,
            "cpu_baseline": cpu_base,
            "parity": parity,
            "parity_8k": parity_8k,
        }
        print(json.dumps(line), flush=True)
    D.ds4sp_destroy(h)


# Same step, other arithmetic choices (config fields), timed for comparison only.
VARIANTS = [
    ("plain_stream_order", dict(dependent_launch=0)),
    ("two_kernel_topk", dict(topk_mode=0)),
    ("indexer_cta_pairs", dict(indexer_kernel=1, topk_mode=0)),
    ("tcgen05_logits", dict(attn_kernel=1)),
    ("ex2_approx_softmax", dict(exp_mode=0)),
    ("fp32_staged_pv", dict(pv_mode=1)),
    ("fp32_staged_pv_ex2_approx", dict(pv_mode=1, exp_mode=0)),
    ("q8_0_cache", dict(kv_format=1)),
    ("q4_0_cache", dict(kv_format=2)),
    ("q8k_q4v_cache", dict(kv_format=3)),
]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-sample", type=int, default=8192)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-verify", action="store_true",
                    help="skip the few-token latency of the 122,880-token verify workload "
                         "and the variants")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the band and 8K prefill lines (and the 8K parity check)")
    ap.add_argument("--soak", type=float, default=1.5,
                    help="seconds of extra steps under the clock sampler")
    ap.add_argument("--topk-mode", type=int, default=1, choices=[0, 1],
                    help="the headline step's top-k form (1, the default = fused indexer + "
                         "top-k; 0 = scores through global memory and a separate top-k "
                         "kernel, also timed in every line for the kernels' own figures)")
    ap.add_argument("--attn-kernel", type=int, default=0, choices=[0, 1],
                    help="the headline step's attention kernel (1 = logits on tcgen05; for "
                         "profiling; the default line uses 0)")
    ap.add_argument("--kv-format", type=int, default=0, choices=[0, 1, 2, 3],
                    help="the headline step's cache format (1 = Q8_0, 2 = Q4_0, 3 = Q8 K / "
                         "Q4 V; for profiling; the default line uses fp16 rows)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
