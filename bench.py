"""Throughput of the L³ forward pass (plan + forward per batch) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl l3|reference]

One step = l3_plan + l3_forward over one batch of the workload (the whole
hot path: sort by token ID, gather-attention, W_up + LayerNorm, W_mix), with
inputs resident in HBM. Rank 0 prints one JSON line.

Multi-GPU (torchrun): every rank runs its own batch of the workload (tokens
are independent, so the batch shards with no collective on the data path);
`value` is all ranks' tokens divided by the slowest rank's time.

--impl reference times the CPU oracle (fp64, all host cores) on bounded
samples of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import static_token_routed_b200 as l3  # noqa: E402
from static_token_routed_b200 import workloads as wl  # noqa: E402

METRIC = "L3 fwd tokens/sec (bf16, 1 B200) and % of roofline (HBM GB/s or tensor-pipe)"
EPS = 1e-5
L2_BYTES = 126 * 2 ** 20
FP32_ALU_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # FFMA lanes x 2 flops x max SM clock


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ----------------------------------------------------------------------------
# algorithmic work (bytes that must move, flops that must be done)
# ----------------------------------------------------------------------------

def algorithmic_work(w: wl.Workload, info) -> dict:
    el = 2 if w.dtype == "bf16" else 4
    n = w.n_tokens
    k_bytes = info.unique_rows_multi * w.d_in * el      # K_t rows read (d_t > 1 groups)
    v_bytes = info.unique_rows * w.d_emb * el           # V_t rows read
    if w.tied:
        # one table: every unique row is read once and serves as key and value
        k_bytes, v_bytes = info.unique_rows * w.d_in * el, 0
    x_bytes = n * w.d_in * el
    y_bytes = n * w.d_out * el
    w_bytes = (w.d_up * w.d_emb + 2 * w.d_up + w.d_out * (w.d_up + w.d_in)) * el
    ids_bytes = n * 4
    total_bytes = k_bytes + v_bytes + x_bytes + y_bytes + w_bytes + ids_bytes
    return {"bytes": total_bytes, "k_bytes": k_bytes, "v_bytes": v_bytes,
            "x_bytes": x_bytes, "y_bytes": y_bytes, "w_bytes": w_bytes,
            "a_bytes": n * w.d_emb * el, "h_bytes": n * w.d_up * el,
            "up_flops": 2 * n * w.d_emb * w.d_up,
            "mix_flops": 2 * n * w.d_out * (w.d_up + w.d_in)}


def attention_flops(ids: np.ndarray, offsets: np.ndarray, w: wl.Workload) -> int:
    d = np.diff(offsets.astype(np.int64))[ids]
    return int(2 * np.sum(d[d > 1]) * (w.d_in + w.d_emb))


# DRAM bytes (read + write) per launch of a kernel, from one ncu capture of
#   ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum
#       --clock-control none -k regex:k_mix_gemm_pair -s 6 -c 4
#       python bench.py --workload <w> --only --steps 3 --warmup 3 --no-e2e --cpu-seconds 0
# keyed by (kernel, workload, tokens), with the digest of the kernel's source
# files at capture time: a figure is reported only while those sources are
# unchanged (source_digest), else traffic is null
TRAFFIC = {
    ("mix_gemm_tc", "paper_shaped", 65536): {"bytes": 618714624 + 246600192,
                                             "sources": ("gemm_tc.cu", "sm100.cuh"),
                                             "digest": "767e851ebfa2ff22", "captured": "2026-12"},
    ("up_z_gemm_tc", "paper_shaped", 65536): {"bytes": 69490944 + 213960960,
                                              "sources": ("gemm_tc.cu", "sm100.cuh"),
                                              "digest": "767e851ebfa2ff22", "captured": "2026-12"},
}


def traffic_for(kernel: str, w) -> dict:
    t = TRAFFIC.get((kernel, w.name, w.n_tokens))
    if t is None:
        return {"traffic": None, "traffic_note": "no ncu capture for this kernel and workload"}
    if t["digest"] is None or source_digest(*t["sources"]) != t["digest"]:
        return {"traffic": None,
                "traffic_note": f"ncu capture of {t['captured']} predates the current "
                                f"{', '.join(t['sources'])}"}
    return {"traffic": t["bytes"], "traffic_note": f"ncu dram read+write per launch, "
                                                   f"captured {t['captured']}"}


# per-kernel roofline: what each kernel must move or compute per launch
def kernel_roofline(name: str, work: dict, attn_flops: int, peaks: dict, tensor_peak: float):
    if name.startswith("attn"):
        bytes_ = work["k_bytes"] + work["v_bytes"] + work["x_bytes"] + work["a_bytes"]
        return "hbm", bytes_, "GB/s", peaks["hbm_gbs"], "HBM copy"
    if name.startswith("up"):
        f = work["up_flops"]
    elif name.startswith("mix"):
        f = work["mix_flops"]
    else:
        return None
    if name.endswith("simt") or name.startswith("up_gemm"):
        return "alu", f, "TFLOP/s", FP32_ALU_PEAK_TFLOPS, "FFMA lanes x max clock"
    return "tensor", f, "TFLOP/s", tensor_peak, "bf16 tensor"


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

REASON_BITS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}


def summarize_clocks(samples):
    """samples: (sm_mhz, sm_max_mhz, reasons bitmask) tuples taken under load."""
    if not samples:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
    reasons = sorted(nm for nm, bit in REASON_BITS.items() if any(r & bit for _, _, r in samples))
    return {"sm_mhz": statistics.median(s for s, _, _ in samples),
            "sm_max_mhz": max(m for _, m, _ in samples), "reasons": reasons,
            "samples": len(samples)}


class ClockSampler:
    """SM clock and clock-event reasons sampled every few ms by NVML (read-only
    queries) on a host thread while the timed region runs."""

    def __init__(self, device: int, period_s: float = 0.005):
        self.device, self.period = device, period_s
        self.samples, self.thread, self.nvml = [], None, None

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = str(getattr(torch.cuda.get_device_properties(self.device), "uuid", "") or "")
            uuid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            h = nv.nvmlDeviceGetHandleByUUID(uuid)
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self.nvml = nv
        except Exception:
            return self
        self.stop = threading.Event()

        def run():
            while True:
                try:
                    self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), mx,
                                         nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
                except Exception:
                    pass
                if self.stop.wait(self.period):
                    return

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join()
        if self.nvml is not None:
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        return summarize_clocks(self.samples)


# ----------------------------------------------------------------------------
# CPU oracle timing (baseline / reference arm)
# ----------------------------------------------------------------------------

def time_oracle_bounded(w, tables, batch, min_seconds: float, chunk: int = 256, seed: int = 0):
    """The oracle on random chunks of the batch until min_seconds of work."""
    n_tok, total, cores, k = 0, 0.0, 1, 0
    while total < min_seconds and n_tok < w.n_tokens:
        n, dt, cores = time_oracle(w, tables, batch, chunk, seed=seed + k)
        n_tok, total, k = n_tok + n, total + dt, k + 1
    return n_tok, total, cores


def time_oracle(w, tables, batch, n_sample: int, seed: int = 0):
    import oracle  # test infrastructure: only the CPU-baseline and reference legs use it
    rng = np.random.default_rng(seed)
    sel = np.sort(rng.choice(w.n_tokens, size=min(n_sample, w.n_tokens), replace=False))
    t0 = time.perf_counter()
    oracle.forward(batch.ids, tables.offsets, batch.x, tables.W_K, tables.W_V, tables.W_up,
                   tables.ln_gamma, tables.ln_beta, tables.W_mix, EPS, select=sel)
    dt = time.perf_counter() - t0
    return len(sel), dt, oracle.threads()


def run_reference(args, w, rank):
    if rank != 0:
        return
    tables, batch = wl.make_tables(w), wl.make_batch(w)
    n_sample = args.ref_sample
    for _ in range(args.warmup):
        time_oracle(w, tables, batch, max(1, n_sample // 8), seed=1)
    total_tok, total_s, cores = 0, 0.0, 1
    for k in range(args.steps):
        n, dt, cores = time_oracle(w, tables, batch, n_sample, seed=100 + k)
        total_tok += n
        total_s += dt
    value = total_tok / total_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, args),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{n_sample} random tokens of the {w.name} batch per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# ranks: each rank plans and runs its own batch; only the timing is reduced
# ----------------------------------------------------------------------------

def rank_workload(base: wl.Workload, rank: int) -> wl.Workload:
    """Same tables on every rank, a different batch per rank (weak scaling)."""
    return wl.with_tokens(base, base.n_tokens, base.batch_seed + 1000 * rank) if rank else base


def max_over_ranks(value: float, dist, device) -> float:
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Tokens of all ranks over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max * 1e-3)


def run_lzw(args, w):
    """Host-side LZW allocation (l3_lzw_allocate) of the workload's vocab / v /
    k on a synthetic phrase-structured Zipf corpus; the plain-Python oracle
    on a prefix of it is the CPU baseline."""
    corpus = wl.zipf_corpus(w.vocab, args.lzw, seed=w.table_seed)
    times = []
    for _ in range(max(1, args.steps)):
        t0 = time.perf_counter()
        d, n_words = l3.l3_lzw_allocate(corpus, w.vocab, w.v, w.k)
        times.append(time.perf_counter() - t0)
    sec = statistics.median(times)
    # the same allocation with the codeword walk on the GPU: host scan plus
    # device walk, wall time per call, and the walk's kernels by CUDA events
    dev_times, walk_ms = [], None
    if torch.cuda.is_available():
        d_dev = torch.empty(w.vocab, dtype=torch.int32, device="cuda")
        l3.l3_lzw_allocate_device(corpus, w.vocab, w.v, w.k, d_dev)  # warm-up
        l3.l3_profile_enable(True)
        for _ in range(max(1, args.steps)):
            t0 = time.perf_counter()
            l3.l3_lzw_allocate_device(corpus, w.vocab, w.v, w.k, d_dev)
            dev_times.append(time.perf_counter() - t0)
        kern = l3.l3_profile_read()
        l3.l3_profile_enable(False)
        walk_ms = sum(t for _, t in kern.values()) / max(1, args.steps)
        assert np.array_equal(d_dev.cpu().numpy(), d), "device walk differs from the host walk"
    from oracle import lzw_allocation  # test infrastructure: CPU-baseline leg only
    n_ref = min(len(corpus), 100_000)
    t0 = time.perf_counter()
    lzw_allocation.allocate(corpus[:n_ref], w.vocab, w.v, w.k)
    ref = time.perf_counter() - t0
    line = {"mode": "lzw_allocation", "metric": "corpus tokens/s through the allocation",
            "value": len(corpus) / sec, "unit": "tokens/s", "higher_is_better": True,
            "seconds": sec, "steps": max(1, args.steps),
            "config": {"workload": w.name, "vocab": w.vocab, "v": w.v, "k": w.k,
                       "corpus_tokens": len(corpus), "corpus": "synthetic phrase-structured Zipf"},
            "codewords": n_words, "tokens_at_k": int((d == w.k).sum()),
            "tokens_at_1": int((d == 1).sum()), "max_d": int(d.max()),
            "device_walk": None if not dev_times else {
                "seconds": statistics.median(dev_times), "walk_kernels_ms": walk_ms,
                "note": "l3_lzw_allocate_device: host corpus scan + GPU walk (bit-identical d_t)"},
            "cpu_baseline": {"value": n_ref / ref, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"first {n_ref} corpus tokens, plain-Python oracle"}}
    print(json.dumps(line), flush=True)


def run_backward(args, w, tables, batch, dev, dist, world, rank):
    """Plan, forward and backward (fp32 gradients for a random dL/dy) per
    batch."""
    d = {k: getattr(tables, k).to(dev) for k in ("offsets", "W_K", "W_up", "ln_gamma", "ln_beta",
                                                 "W_mix")}
    d["W_V"] = d["W_K"] if tables.W_V is tables.W_K else tables.W_V.to(dev)
    ids_d, x_d = batch.ids.to(dev), batch.x.to(dev)
    y_d = torch.empty(w.n_tokens, w.d_out, dtype=w.torch_dtype, device=dev)
    g = torch.Generator(device=dev).manual_seed(0)
    dy = torch.randn(w.n_tokens, w.d_out, generator=g, device=dev).to(w.torch_dtype)
    dims = l3.make_dims(w.vocab, w.v, w.k, w.d_in, w.d_emb, w.d_up, w.d_out, w.torch_dtype, EPS)
    stream = torch.cuda.current_stream(dev)

    def step():
        plan = l3.l3_plan(ids_d, d["offsets"], dims, stream)
        l3.l3_forward(x_d, plan, d["W_K"], d["W_V"], d["W_up"], d["ln_gamma"], d["ln_beta"],
                      d["W_mix"], y_d, stream)
        grads = l3.l3_backward(x_d, plan, d["W_K"], d["W_V"], d["W_up"], d["ln_gamma"],
                               d["ln_beta"], d["W_mix"], dy, stream)
        return plan, grads

    for _ in range(max(3, args.warmup)):
        p, _ = step()
        p.destroy()
    l3.l3_profile_enable(True)
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        p, _ = step()
        p.destroy()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    kernels = l3.l3_profile_read()
    l3.l3_profile_enable(False)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dist, dev)
    if rank != 0:
        return
    bwd_ms = sum(t for k, (_, t) in kernels.items() if k.startswith("bwd")) / args.steps
    line = {"metric": METRIC, "mode": "forward+backward", "value": job_throughput(w.n_tokens, world, ms),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "backward_ms_per_step": bwd_ms, "higher_is_better": True,
            "scaling": "weak", "dtype": "bf16" if w.dtype == "bf16" else "fp32",
            "data": "synthetic", "config": config_of(w, args),
            "kernels": {k: {"launches": nl, "per_step_ms": t / args.steps}
                        for k, (nl, t) in kernels.items()}}
    print(json.dumps(line), flush=True)


def run_offload(args, w, tables, batch, dev, dist, world, rank):
    """Tables in pinned host memory: each step plans the batch (l3_plan_staged),
    copies its rows across PCIe into device staging tables (l3_stage_rows) and
    runs l3_forward on them. Staging of batch i+1 overlaps the forward of i."""
    d = {k: getattr(tables, k).to(dev) for k in ("offsets", "W_up", "ln_gamma", "ln_beta",
                                                 "W_mix")}
    WK = tables.W_K.pin_memory()
    WV = WK if tables.W_V is tables.W_K else tables.W_V.pin_memory()
    ids_d, x_d = batch.ids.to(dev), batch.x.to(dev)
    y_d = torch.empty(w.n_tokens, w.d_out, dtype=w.torch_dtype, device=dev)
    dims = l3.make_dims(w.vocab, w.v, w.k, w.d_in, w.d_emb, w.d_up, w.d_out, w.torch_dtype, EPS)
    stream, side = torch.cuda.current_stream(dev), torch.cuda.Stream(dev)
    staged_ev = [torch.cuda.Event(), torch.cuda.Event()]
    done = [torch.cuda.Event(), torch.cuda.Event()]
    n = [0]

    def step():
        k = n[0]
        if k >= 2:
            done[k % 2].synchronize()
        plan = l3.l3_plan(ids_d, d["offsets"], dims, side, staged=True)
        rows = plan.info().unique_rows
        with torch.cuda.stream(side):
            Ks = torch.empty(rows, w.d_in, dtype=w.torch_dtype, device=dev)
            Vs = torch.empty(rows, w.d_emb, dtype=w.torch_dtype, device=dev)
        l3.l3_stage_rows(plan, WK, WV, Ks, Vs, side)
        staged_ev[k % 2].record(side)
        stream.wait_event(staged_ev[k % 2])
        l3.l3_forward(x_d, plan, Ks, Vs, d["W_up"], d["ln_gamma"], d["ln_beta"], d["W_mix"], y_d,
                      stream)
        Ks.record_stream(stream)
        Vs.record_stream(stream)
        done[k % 2].record(stream)
        n[0] = k + 1
        return plan

    for _ in range(max(3, args.warmup)):
        step().destroy()
    p0 = step()
    l3.l3_forward_status(p0)
    rows = p0.info().unique_rows
    p0.destroy()
    l3.l3_profile_enable(True)
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index or 0) as clocks:
        ev0.record(stream)
        side.wait_event(ev0)
        for _ in range(args.steps):
            step().destroy()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    kernels = l3.l3_profile_read()
    l3.l3_profile_enable(False)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dist, dev)
    if rank != 0:
        return
    el = 2 if w.dtype == "bf16" else 4
    staged_bytes = rows * (w.d_in + w.d_emb) * el
    line = {"metric": METRIC, "mode": "offload", "value": job_throughput(w.n_tokens, world, ms),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "dtype": "bf16" if w.dtype == "bf16" else "fp32", "data": "synthetic",
            "config": dict(config_of(w, args), tables="pinned host memory"),
            "clocks": clocks.summary(),
            "staged_rows_per_step": rows, "staged_bytes_per_step_max": staged_bytes,
            "host_link_GBps": staged_bytes / (ms * 1e-3) / 1e9,
            "kernels": {k: {"launches": nl, "per_step_ms": t / args.steps}
                        for k, (nl, t) in kernels.items()}}
    print(json.dumps(line), flush=True)


def config_of(w, args):
    return {"workload": w.name, "global_batch": w.n_tokens * args.gpus, "tokens_per_gpu": w.n_tokens,
            "vocab": w.vocab, "v": w.v, "k": w.k, "d_in": w.d_in, "d_emb": w.d_emb,
            "d_up": w.d_up, "d_out": w.d_out, "alloc": w.alloc, "ids": w.ids, "tied": w.tied,
            "parallelism": f"dp{args.gpus}",
            "l2": "no flush: per-step working set (W_K/W_V rows, x, y, weights) >> 126 MB L2"}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def tensor_peak(peaks: dict, timed_s: float, clocks: dict):
    """The bf16 tensor peak that applies to this timed region: the burst
    figure (a kernel timed on its own at full clock) unless the region ran
    for seconds with the SM clock well below its maximum, as in the
    sustained measurement."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    slowed = mhz is not None and mx and mhz < 0.9 * mx
    if timed_s >= 2.0 and slowed:
        return peaks["bf16_tflops_sustained"], "sustained"
    return peaks["bf16_tflops"], "burst"


def source_digest(*names: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for nm in names:
        with open(os.path.join(ROOT, "static_token_routed_b200", "csrc", nm), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measure(w, args, dev, dist, world, rank, steps, warmup, with_e2e=True, with_fwd_only=True,
            cpu_seconds=0.0):
    """Time plan + forward of workload `w` (every rank its own batch); returns
    the fields of the JSON line for it (rank 0) or None."""
    tables, batch = wl.make_tables(w), wl.make_batch(w)
    d = {k: getattr(tables, k).to(dev) for k in ("offsets", "W_K", "W_up", "ln_gamma",
                                                 "ln_beta", "W_mix")}
    # a tied workload passes one device table as keys and values
    d["W_V"] = d["W_K"] if tables.W_V is tables.W_K else tables.W_V.to(dev)
    ids_d, x_d = batch.ids.to(dev), batch.x.to(dev)
    y_d = torch.empty(w.n_tokens, w.d_out, dtype=w.torch_dtype, device=dev)
    dims = l3.make_dims(w.vocab, w.v, w.k, w.d_in, w.d_emb, w.d_up, w.d_out, w.torch_dtype, EPS)
    stream = torch.cuda.current_stream(dev)
    # l3_plan synchronises only its own stream: with the plan of batch i+1 on
    # its own stream it runs while batch i's forward is still on the GPU, as in
    # a pipeline over batches.
    plan_stream = torch.cuda.Stream(dev)
    # at most two forwards in flight: before planning batch i+1 the host waits
    # for batch i-1's forward, so the plan memory it freed is reusable
    done = [torch.cuda.Event(), torch.cuda.Event()]
    n_step = [0]

    def step(ids_t, x_t, y_t):
        k = n_step[0]
        if k >= 2:
            done[k % 2].synchronize()
        plan = l3.l3_plan(ids_t, d["offsets"], dims, plan_stream)
        l3.l3_forward(x_t, plan, d["W_K"], d["W_V"], d["W_up"], d["ln_gamma"], d["ln_beta"],
                      d["W_mix"], y_t, stream)
        done[k % 2].record(stream)
        n_step[0] = k + 1
        return plan

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(max(3, warmup)):
        step(ids_d, x_d, y_d).destroy()
    plan0 = step(ids_d, x_d, y_d)
    l3.l3_forward_status(plan0)
    info = plan0.info()
    plan0.destroy()

    # ---- timed region: K steps, plan + forward, device-timed ----
    # per-kernel CUDA events on the forward's launches (the plan's are not
    # timed: their events cost host time in the loop and they are never the
    # dominant kernel)
    l3.l3_profile_enable(2)
    barrier()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index or 0) as clocks:
        ev0.record(stream)
        plan_stream.wait_event(ev0)
        for _ in range(steps):
            step(ids_d, x_d, y_d).destroy()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    kernels = l3.l3_profile_read()
    l3.l3_profile_enable(False)
    ms_max = max_over_ranks(ev0.elapsed_time(ev1) / steps, dist, dev)
    value = job_throughput(w.n_tokens, world, ms_max)
    clock_summary = clocks.summary()

    # ---- end to end through the public API with host buffers ----
    # Each step copies its batch (ids, x) from pinned host memory and reads y
    # back. The copies run on their own streams into two sets of device
    # buffers, so batch i+1 moves over PCIe while batch i computes and batch
    # i-1's y comes back, as in a serving pipeline.
    e2e = None
    if with_e2e:
        ids_h = batch.ids.pin_memory()
        x_h = batch.x.pin_memory()
        y_h = [torch.empty(w.n_tokens, w.d_out, dtype=w.torch_dtype).pin_memory()
               for _ in range(2)]
        ids_s = [torch.empty_like(ids_d) for _ in range(2)]
        x_s = [torch.empty_like(x_d) for _ in range(2)]
        y_s = [torch.empty_like(y_d) for _ in range(2)]
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]  # noqa: E731
        in_ready, fwd_done, out_done = ev(), ev(), ev()
        n_e2e = [0]

        def e2e_step():
            k = n_e2e[0]
            j = k % 2
            if k >= 2:
                h2d.wait_event(fwd_done[j])       # forward k-2 no longer reads slot j
            with torch.cuda.stream(h2d):
                ids_s[j].copy_(ids_h, non_blocking=True)
                x_s[j].copy_(x_h, non_blocking=True)
            in_ready[j].record(h2d)
            plan_stream.wait_event(in_ready[j])
            stream.wait_event(in_ready[j])
            if k >= 2:
                stream.wait_event(out_done[j])    # y of step k-2 has left slot j
            p = step(ids_s[j], x_s[j], y_s[j])
            fwd_done[j].record(stream)
            d2h.wait_event(fwd_done[j])
            with torch.cuda.stream(d2h):
                y_h[j].copy_(y_s[j], non_blocking=True)
            out_done[j].record(d2h)
            n_e2e[0] = k + 1
            return p

        for _ in range(3):
            e2e_step().destroy()
        barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for st in (plan_stream, h2d, d2h):
            st.wait_event(e0)
        for _ in range(steps):
            e2e_step().destroy()
        last = torch.cuda.Event()
        last.record(d2h)
        stream.wait_event(last)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1) / steps, dist, dev)
        e2e = {"value": job_throughput(w.n_tokens, world, ems), "unit": "tokens/s",
               "h2d_bytes_per_step": int(ids_h.numel() * 4 + x_h.numel() * x_h.element_size()),
               "d2h_bytes_per_step": int(y_h[0].numel() * y_h[0].element_size()),
               "copies": "own streams, double-buffered: overlap the previous and next steps"}

    # ---- forward alone: one plan, K forwards (the sort done ahead of time) ----
    fwd_only = None
    if with_fwd_only:
        plan_f = l3.l3_plan(ids_d, d["offsets"], dims, stream)
        for _ in range(3):
            l3.l3_forward(x_d, plan_f, d["W_K"], d["W_V"], d["W_up"], d["ln_gamma"],
                          d["ln_beta"], d["W_mix"], y_d, stream)
        barrier()
        torch.cuda.synchronize(dev)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(steps):
            l3.l3_forward(x_d, plan_f, d["W_K"], d["W_V"], d["W_up"], d["ln_gamma"],
                          d["ln_beta"], d["W_mix"], y_d, stream)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        l3.l3_forward_status(plan_f)
        plan_f.destroy()
        barrier()
        fwd_ms = max_over_ranks(f0.elapsed_time(f1) / steps, dist, dev)
        fwd_only = {"value": job_throughput(w.n_tokens, world, fwd_ms), "unit": "tokens/s",
                    "ms_per_step": fwd_ms, "note": "l3_forward alone on a plan built ahead of time"}

    if rank != 0:
        return None

    # ---- roofline ----
    peaks = load_peaks()
    tpeak, regime = tensor_peak(peaks, ms_max * 1e-3 * steps, clock_summary)
    work = algorithmic_work(w, info)
    attn_flops = attention_flops(batch.ids.numpy(), tables.offsets.numpy(), w)
    total_flops = attn_flops + work["up_flops"] + work["mix_flops"]
    if w.dtype == "bf16":
        t_flop = total_flops / (tpeak * 1e12)
        flop_note = f"bf16 {tpeak} TFLOP/s ({regime})"
    else:
        t_flop = total_flops / (FP32_ALU_PEAK_TFLOPS * 1e12)
        flop_note = f"fp32 FFMA {FP32_ALU_PEAK_TFLOPS:.1f} TFLOP/s (148 SMs x 128 lanes x 2 x 1965 MHz)"
    t_mem = work["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_roof = max(t_mem, t_flop)
    step_roof = {"t_mem_us": t_mem * 1e6, "t_flop_us": t_flop * 1e6,
                 "bound": "hbm" if t_mem > t_flop else ("tensor" if w.dtype == "bf16" else "alu"),
                 "frac": t_roof / (ms_max * 1e-3), "alg_bytes": work["bytes"],
                 "alg_flops": total_flops,
                 "peak_note": f"{peaks['source']}: HBM {peaks['hbm_gbs']} GB/s, {flop_note}"}
    kern = {k: {"launches": n, "total_ms": t, "per_step_ms": t / steps}
            for k, (n, t) in kernels.items()}
    # the dominant kernel of the forward: plan kernels run on their own stream
    # beside the previous batch's forward, so their event times include
    # waiting for SMs and say nothing about their own speed
    fwd = {k: v for k, v in kernels.items()
           if kernel_roofline(k, work, attn_flops, peaks, tpeak) is not None}
    top = max(fwd.items(), key=lambda kv: kv[1][1])[0] if fwd else None
    roof = None
    if top is not None:
        kr = kernel_roofline(top, work, attn_flops, peaks, tpeak)
        n_launch, tot_ms = kernels[top]
        if kr is not None:
            bound, units, unit, peak, peak_src = kr
            per_launch_s = tot_ms * 1e-3 / n_launch
            launches_per_step = n_launch / steps
            per_launch_units = units / launches_per_step
            achieved = per_launch_units / per_launch_s / (1e9 if unit == "GB/s" else 1e12)
            roof = {"kernel": top, "bound": bound, "achieved": achieved, "peak": peak,
                    "unit": unit, "frac": achieved / peak,
                    "peak_source": f"{peaks['source']} ({peak_src})"}
            roof.update(traffic_for(top, w))

    # ---- CPU baseline: the oracle on a bounded sample ----
    cpu = None
    if world == 1 and cpu_seconds > 0:
        n_s, dt, cores = time_oracle_bounded(w, tables, batch, cpu_seconds,
                                             chunk=min(256, w.n_tokens))
        cpu = {"value": n_s / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n_s} random tokens of the {w.name} batch in chunks of "
                         f"{min(256, w.n_tokens)} (fp64 oracle, {dt:.1f} s)"}
        if w.n_tokens <= 4096:
            # small batches: the whole batch on one host thread as well
            import oracle  # test infrastructure: CPU-baseline leg only
            t0 = time.perf_counter()
            oracle.forward(batch.ids, tables.offsets, batch.x, tables.W_K, tables.W_V, tables.W_up,
                           tables.ln_gamma, tables.ln_beta, tables.W_mix, EPS, n_threads=1)
            cpu["single_thread"] = {"value": w.n_tokens / (time.perf_counter() - t0),
                                    "unit": "tokens/s", "sample": "the whole batch"}

    return {"value": value, "ms_per_step": ms_max, "steps": steps, "warmup": warmup,
            "dtype": "bf16" if w.dtype == "bf16" else "fp32", "config": config_of(w, args),
            "clocks": clock_summary, "e2e": e2e,
            "gpu_launches": int(sum(n for n, _ in kernels.values())),
            "roofline": roof, "step_roofline": step_roof, "kernels": kern,
            "cpu_baseline": cpu, "forward_only": fwd_only,
            "plan": {"groups": info.n_groups, "dense_groups": info.n_dense_groups,
                     "dense_tiles": info.n_dense_tiles, "tail_items": info.n_tail_items,
                     "unique_rows": info.unique_rows}}


# the benchmark's other synthetic workloads besides the headline, each measured in the same run
OTHER_WORKLOADS = ("tiny_fp32", "small_bf16", "decode", "dense_stress", "uniform")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="paper_shaped", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="l3", choices=["l3", "reference"])
    ap.add_argument("--ref-sample", type=int, default=256, help="oracle tokens per reference step")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="seconds of oracle work for cpu_baseline (0: skip)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="tokens per rank (default: the workload's batch size)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", action="store_true",
                    help="measure the named workload alone (no per_workload lines)")
    ap.add_argument("--lzw", type=int, default=0, metavar="TOKENS",
                    help="time the LZW allocation on a synthetic corpus of this many tokens")
    ap.add_argument("--backward", action="store_true",
                    help="time l3_forward + l3_backward per batch")
    ap.add_argument("--offload", action="store_true",
                    help="W_K / W_V in pinned host memory; each step stages the batch's rows")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    base = wl.WORKLOADS[args.workload]
    if args.tokens > 0:
        base = wl.with_tokens(base, args.tokens)

    if args.impl == "reference":
        run_reference(args, base, rank)
        return
    if args.lzw:
        if rank == 0:
            run_lzw(args, base)
        return

    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    # each rank: same tables, its own batch
    w = rank_workload(base, rank)
    if args.offload or args.backward:
        tables, batch = wl.make_tables(w), wl.make_batch(w)
        (run_offload if args.offload else run_backward)(args, w, tables, batch, dev, dist, world,
                                                        rank)
        return

    head = measure(w, args, dev, dist, world, rank, args.steps, args.warmup,
                   with_e2e=not args.no_e2e, with_fwd_only=True, cpu_seconds=args.cpu_seconds)
    per_workload = None
    if world == 1 and not args.only and args.tokens == 0 and args.workload == "paper_shaped":
        # the other synthetic workloads at one GPU: shorter CPU samples, the
        # same steps (each step is shorter than the headline's)
        torch.cuda.empty_cache()
        per_workload = {}
        for name in OTHER_WORKLOADS:
            r = measure(wl.WORKLOADS[name], args, dev, dist, world, rank, args.steps,
                        args.warmup, with_e2e=False, with_fwd_only=True,
                        cpu_seconds=min(3.0, args.cpu_seconds))
            torch.cuda.empty_cache()
            per_workload[name] = {k: r[k] for k in ("value", "ms_per_step", "dtype", "config",
                                                    "clocks", "roofline", "step_roofline",
                                                    "cpu_baseline", "forward_only", "plan",
                                                    "gpu_launches", "kernels")}
    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return
    line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": head["dtype"], "data": "synthetic", "config": head["config"],
            "clocks": head["clocks"], "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
            "roofline": head["roofline"], "step_roofline": head["step_roofline"],
            "kernels": head["kernels"], "cpu_baseline": head["cpu_baseline"],
            "forward_only": head["forward_only"],
            "pipelining": "batch i+1's l3_plan on its own stream overlaps batch i's l3_forward",
            "plan": head["plan"]}
    if per_workload is not None:
        line["per_workload"] = per_workload
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
