"""Benchmark of the Infini-attention layer forward on B200.

One step = one infini_attn_forward over one batch of the workload (local
attention, retrieval, gate and memory update for every segment), inputs
resident in HBM.  Prints one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

Multi-GPU (launched by torchrun, one process per GPU): the work shards over
independent (batch, KV head) chains with no data-path collective.  By default
every rank runs its own full batch of the workload (weak scaling) and the
value is all ranks' tokens over the slowest rank's device time; with
``--shard chains`` the workload's own chains are split into one (batch rows x
KV heads) block per rank (strong scaling: the value is the workload's tokens
over the slowest rank's device time).

``--impl reference`` times the float64 CPU oracle on a bounded sample of the
same workload, on the host cores.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from compressive_memory_transformer_segment_b200 import configs, synth  # noqa: E402

METRIC = "Infini-attention fwd tokens/s on 1 B200; % of bf16 tensor-core peak"
DEFAULT_CONFIG = "8b-delta"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one attention
# launch, from an ncu capture summarised under profiles/, valid only while the
# kernel sources hash to what they were at capture time.
ATTENTION_TRAFFIC = {
    "8b-delta": {"bytes": 2 * (409.388544e6 + 231.382016e6),
                 "note": "ncu capture at batch 1, scaled x2 to the batch-2 launch",
                 "profile": "profiles/tc_attention_8b-delta.md",
                 "sha1": {"tc_attention.cu": "6370c59817bbe2487940b477ce95a2cbc7277627",
                          "tc_common.cuh": "a896981e1b8e14dfabfd0f26a799d64c0af65a34"}},
    "1m-linear": {"bytes": 16 * (1.754910e9 + 0.5212416e9),
                  "note": "ncu capture of the same shape cut to 65,536 tokens, scaled x16 to the "
                          "1,048,576-token launch (traffic grows with the tokens)",
                  "profile": "profiles/tc_attention_1m-linear.md",
                  "sha1": {"tc_attention.cu": "6370c59817bbe2487940b477ce95a2cbc7277627",
                           "tc_common.cuh": "a896981e1b8e14dfabfd0f26a799d64c0af65a34"}},
}


# The same for the projection prologue's qkv_rope launch.
PROJECTION_TRAFFIC = {
    "8b-delta": {"bytes": 2 * (792.638720e6 + 388.922880e6),
                 "note": "ncu capture at batch 1, scaled x2 to the batch-2 launch (traffic grows "
                         "with the token rows)",
                 "profile": "profiles/qkv_rope_8b-projection.md",
                 "sha1": {"qkv_rope.cu": "6f1d6c92e520d53cb8aa0da4741bfc9c36993ebb",
                          "tc_common.cuh": "a896981e1b8e14dfabfd0f26a799d64c0af65a34"}},
}


def attention_traffic(name, table=None):
    """Recorded per-launch traffic for this workload, or None if the kernel
    changed since the counters were taken (or none were taken)."""
    import hashlib
    rec = (ATTENTION_TRAFFIC if table is None else table).get(name)
    if rec is None:
        return None
    csrc = os.path.join(ROOT, "compressive_memory_transformer_segment_b200", "csrc")
    for fn, sha in rec["sha1"].items():
        with open(os.path.join(csrc, fn), "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != sha:
                return None
    return rec


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---------------------------------------------------------------- oracle timing

def oracle_sample(w, budget_s):
    """Time the float64 oracle on whole KV chains (each with all query heads of
    its group), segment by segment, until about ``budget_s`` seconds have passed.

    Returns (token-equivalents/s, description, seconds).  One token of the
    workload needs all H_kv chains, so r rows of one chain count as r/H_kv tokens.
    """
    import oracle  # the CPU baseline is the only product-adjacent use of the oracle

    g = w.H_q // w.H_kv
    beta = synth.make_beta(w)
    chains = [(b, j) for b in range(w.B) for j in range(w.H_kv)]
    rows = 0
    nseg = 0
    used = []
    elapsed = 0.0
    for b, j in chains:
        kc = synth.as_float64(synth.make_head(w, "k", b, j), w.dtype)
        vc = synth.as_float64(synth.make_head(w, "v", b, j), w.dtype)
        heads = range(j * g, (j + 1) * g)
        qs = {h: synth.as_float64(synth.make_head(w, "q", b, h), w.dtype) for h in heads}
        used.append((b, j))
        t0 = time.perf_counter()
        scan = oracle.scan_states(kc, vc, np.zeros((w.d_k, w.d_v)), np.zeros(w.d_k),
                                  w.seg_len, w.rule)
        for s, r0, r1, M, z in scan:
            if r0 == r1:
                break
            for h in heads:
                oracle.segment_output(qs[h][r0:r1], kc[r0:r1], vc[r0:r1], M, z, float(beta[h]))
            rows += r1 - r0
            nseg += 1
            if elapsed + time.perf_counter() - t0 >= budget_s:
                next(scan)  # the generator applies this segment's memory update on resume
                break
        elapsed += time.perf_counter() - t0
        if elapsed >= budget_s:
            break
    tokens = rows / w.H_kv
    desc = (f"oracle (NumPy float64), {len(used)} (batch, KV head) chain(s) from {used[0]}, "
            f"each with its {g} query head(s): {nseg} segment(s) of up to {w.seg_len} rows "
            f"({rows} rows) in {elapsed:.2f} s of compute (input generation untimed); "
            f"token-equivalents = rows / H_kv")
    return tokens / elapsed, desc, elapsed


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    budget = max(1.0, args.reference_budget / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, budget)
    vals, descs, times = [], [], []
    for _ in range(args.steps):
        v, d, dt = oracle_sample(w, budget)
        vals.append(v)
        descs.append(d)
        times.append(dt)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * statistics.median(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, args.gpus, None),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": host_cores(),
                         "kind": "oracle", "sample": descs[-1]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm

class ClockSampler:
    """Samples SM clock and throttle reasons while the timed region runs.

    Uses NVML in a background thread (every 10 ms); falls back to an
    nvidia-smi subprocess.  Only reads GPU state."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.thread = None
        self.proc = None
        # Raw samples of the nvidia-smi fallback (INFINI_CLOCKS_DIR, else the
        # temporary directory).
        import tempfile
        out_dir = os.environ.get("INFINI_CLOCKS_DIR", tempfile.gettempdir())
        self.path = os.path.join(out_dir, f"clocks_rank{gpu_index}.csv")

    def _nvml_loop(self, pynvml, h):
        bits = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
                "sw_power_cap": 0x4}
        while not self.stop:
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, smax, [n for n, b in bits.items() if r & b]))
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        self.stop = False
        try:
            import threading
            import pynvml
            pynvml.nvmlInit()
            idx = self.gpu
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                try:
                    idx = int(vis.split(",")[self.gpu])
                except (ValueError, IndexError):
                    pass
            h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.thread = threading.Thread(target=self._nvml_loop, args=(pynvml, h), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu),
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.stop = True
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm, smax = float(parts[1]), float(parts[2])
                except ValueError:
                    continue
                rs = [n for n, flag in zip(self.NAMES, parts[5:9]) if flag.lower().startswith("active")]
                self.samples.append((sm, smax, rs))

    def summary(self):
        if not self.samples:
            return None
        sm = [x[0] for x in self.samples]
        reasons = sorted({r for x in self.samples for r in x[2]})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[1] for x in self.samples),
                "reasons": reasons, "samples": len(sm),
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


def config_dict(w, n_gpus, l2_note, block=None):
    d = {"workload": w.name, "B": w.B, "H_q": w.H_q, "H_kv": w.H_kv, "L": w.L,
         "d_k": w.d_k, "d_v": w.d_v, "seg_len": w.seg_len, "T": w.T, "rule": w.rule,
         "io_dtype": w.dtype, "state_dtype": "f32", "tokens_per_step_per_gpu": w.tokens,
         "parallelism": f"dp{n_gpus} (independent (batch, KV head) chains, no collective)"}
    if block is not None:
        b0, b1, h0, h1 = block
        d["tokens_per_step_per_gpu"] = None
        d["parallelism"] = (f"chains{n_gpus} (the workload's (batch row, KV head) chains split "
                            f"into one block per rank, no collective; rank 0: rows [{b0}, {b1}), "
                            f"KV heads [{h0}, {h1}))")
    if l2_note:
        d["l2"] = l2_note
    return d


def run_gpu(args, w):
    import torch
    import torch.distributed as dist

    from compressive_memory_transformer_segment_b200 import api, shard

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    api.load_library()
    # --shard chains: this rank runs only its block of the workload's (batch
    # row, KV head) chains (strong scaling); otherwise every rank runs the
    # whole workload on inputs of its own (weak scaling).
    w_job, block = w, None
    if args.shard == "chains":
        block = shard.chain_block(w.B, w.H_kv, world, rank)
        g = w.H_q // w.H_kv
        b0, b1, h0, h1 = block
        w = w.with_(B=b1 - b0, H_kv=h1 - h0, H_q=(h1 - h0) * g)
    job_tokens = w_job.tokens if block is not None else w.tokens * world

    def barrier():
        if world > 1:
            dist.barrier()

    # Inputs: seeded, generated on the host, copied once to HBM.
    wr = w.with_(seed=w.seed + 7919 * rank)
    inp = synth.make_inputs(wr)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def host_tensor(x):
        if w.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))

    hq, hk, hv = (host_tensor(inp[n]) for n in ("q", "k", "v"))
    q, k, v = (t.to(dev) for t in (hq, hk, hv))
    beta = torch.from_numpy(inp["beta"]).to(dev)
    M0, z0 = api.init_state(w.B, w.H_kv, w.d_k, w.d_v, device=dev)
    out = torch.empty((w.B, w.H_q, w.L, w.d_v), dtype=tdt, device=dev)
    M1 = torch.empty_like(M0)
    z1 = torch.empty_like(z0)
    dims = api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, tdt)
    plan = api.plan(dims, w.seg_len, w.rule)
    ws = torch.empty(plan["workspace_bytes"], dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
    flush = None
    if in_bytes < 2 * L2_BYTES:
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        l2_note = "L2 flushed (256 MiB write) between timed steps; each step timed alone"
    else:
        l2_note = f"inputs ({in_bytes / 2**20:.0f} MiB) larger than L2; steps timed back to back"

    def step():
        api.forward(q, k, v, beta, M0, z0, w.seg_len, w.rule, out=out, M_out=M1, z_out=z1,
                    workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    api.sync_status(stream)

    def timed_pass(n, flush_each):
        """Device time of n steps (each alone after an L2 flush, or back to back)."""
        if not flush_each:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            return e0.elapsed_time(e1)
        total = 0.0
        for _ in range(n):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            total += e0.elapsed_time(e1)
        return total

    # Per-kernel device times come from a separate pass with events around the
    # state scan and the attention: those events sit between the kernels and
    # would add their own gaps to the timed steps.
    api.set_kernel_timing(True)
    api.kernel_times(reset=True)
    timed_pass(args.steps, flush is not None)
    api.set_kernel_timing(False)
    ktimes = api.kernel_times(reset=True)
    api.sync_status(stream)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        elapsed_ms = timed_pass(args.steps, flush is not None)
    barrier()
    torch.cuda.synchronize(dev)
    api.sync_status(stream)

    max_ms = shard.max_over_ranks(elapsed_ms, device=dev)
    tokens = job_tokens * args.steps
    value = tokens / (max_ms / 1000.0)

    # End to end through the C ABI with host buffers (pinned), copies inside.
    if not args.e2e:
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": "tokens/s",
                              "ms_per_step": max_ms / args.steps,
                              "kernel_ms": {k: v[0] / max(v[1], 1) for k, v in ktimes.items()},
                              "config": config_dict(w_job, world, l2_note, block),
                              "note": "profiling run"}))
        return 0
    hq_p, hk_p, hv_p = (x.pin_memory() for x in (hq, hk, hv))
    hbeta = torch.from_numpy(inp["beta"]).pin_memory()
    hM0 = torch.zeros(M0.shape, dtype=torch.float32).pin_memory()
    hz0 = torch.zeros(z0.shape, dtype=torch.float32).pin_memory()
    hout = torch.empty(out.shape, dtype=tdt).pin_memory()
    hM1 = torch.empty(M0.shape, dtype=torch.float32).pin_memory()
    hz1 = torch.empty(z0.shape, dtype=torch.float32).pin_memory()
    arena = torch.empty(api.host_arena_bytes(dims, w.seg_len, w.rule), dtype=torch.uint8, device=dev)
    del ws
    e2e_steps = max(1, min(args.steps, 5))

    def e2e_step():
        api.forward_host(hq_p, hk_p, hv_p, hbeta, hM0, hz0, w.seg_len, w.rule, hout, hM1, hz1,
                         arena, stream=stream)

    e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = shard.max_over_ranks(e0.elapsed_time(e1), device=dev)
    e2e_value = job_tokens * e2e_steps / (e2e_ms / 1000.0)
    h2d = sum(x.numel() * x.element_size() for x in (hq_p, hk_p, hv_p, hbeta, hM0, hz0))
    d2h = sum(x.numel() * x.element_size() for x in (hout, hM1, hz1))

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    flops = configs.algorithmic_flops(w)
    att_ms, att_n = ktimes["attention"]
    scan_ms, scan_n = ktimes["state_scan"]
    # Dominant kernel: the segment attention kernel (local attention, retrieval,
    # gate).  Its algorithmic flops: every flop of the step except the update.
    upd = w.B * w.H_kv * w.L * (2 * w.d_k * w.d_v + w.d_k)
    if w.rule == "delta":
        upd += w.B * w.H_kv * w.L * (2 * w.d_k * w.d_v + 2 * w.d_k)
    att_flops = flops - upd
    att_avg_s = (att_ms / max(att_n, 1)) / 1000.0
    achieved = att_flops / att_avg_s / 1e12 if att_avg_s > 0 else 0.0
    peak = peaks["bf16_tflops"]
    step_ms = max_ms / args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "strong" if block is not None else "weak",
        "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded Philox N(0,1) q/k/v, U(-r,r) beta)",
        "config": config_dict(w_job, world, l2_note, block),
        "path": plan["path"],
        "tc_peak_frac_step": (flops / (step_ms / 1000.0)) / (peak * 1e12),
        # The step's algorithmic bytes (q, k, v read once, out written once,
        # M/z in and out) against the measured HBM copy bandwidth.
        "hbm_frac_step": (configs.algorithmic_bytes(w) / (step_ms / 1000.0)) / (peaks["hbm_gbs"] * 1e9),
        "clocks": clocks.summary(),
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": plan["launches"] * args.steps,
        "roofline": {"bound": "tensor", "kernel": "segment attention", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peak_src} bf16 burst",
                     "traffic": (attention_traffic(w.name) or {}).get("bytes"),
                     "traffic_note": (attention_traffic(w.name) or {}).get("note"),
                     "algorithmic_flops_per_launch": att_flops,
                     "avg_launch_ms": att_avg_s * 1000.0},
        "kernel_ms": {"attention": att_ms / max(att_n, 1), "state_scan": scan_ms / max(scan_n, 1)},
    }
    if args.cpu_baseline:
        v, desc, _ = oracle_sample(w_job, args.cpu_budget)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": host_cores(),
                                "kind": "oracle", "sample": desc}
    print(json.dumps(line), flush=True)
    return 0


def run_seq_parallel(args, w):
    """Sequence-parallel linear rule (strong scaling): the workload's sequence
    is cut into one run of whole segments per rank (shard.segment_range); each
    rank's timed step is its run's state update from zero, one all-gather of
    the updates, the exclusive prefix and the forward over its run."""
    import torch
    import torch.distributed as dist

    from compressive_memory_transformer_segment_b200 import api, shard

    if w.rule != "linear":
        raise SystemExit("--seq-parallel needs a linear-rule workload (the delta rule is sequential)")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    api.load_library()
    l0, l1 = shard.segment_range(w.L, w.seg_len, world, rank)
    # This rank's rows only, drawn with a seed of their own (the values differ
    # from one draw of the whole sequence; the throughput does not depend on
    # them), without the inserted key/value pair.
    inp = synth.make_inputs(w.with_(L=l1 - l0, seed=w.seed + 104729 * (l0 // w.seg_len),
                                    insert_pair=False))
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def dev_tensor(x):
        if w.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dev)

    q, k, v = (dev_tensor(inp[n]) for n in ("q", "k", "v"))
    beta = torch.from_numpy(inp["beta"]).to(dev)
    M0, z0 = api.init_state(w.B, w.H_kv, w.d_k, w.d_v, device=dev)

    def step():
        return shard.sequence_parallel_forward(q, k, v, beta, M0, z0, w.seg_len,
                                               forward=api.forward, state_update=api.state_update,
                                               state_sum=api.state_sum)

    for _ in range(args.warmup):
        step()
    api.sync_status()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    with ClockSampler(local) as clocks:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    api.sync_status()
    max_ms = shard.max_over_ranks(e0.elapsed_time(e1), device=dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    tokens = w.B * w.L * args.steps
    step_ms = max_ms / args.steps
    peaks, _ = load_peaks()
    flops = configs.algorithmic_flops(w)
    print(json.dumps({
        "metric": "Infini-attention fwd tokens/s, sequence-parallel linear rule",
        "value": tokens / (max_ms / 1000.0), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded Philox N(0,1) q/k/v, U(-r,r) beta)",
        "config": {"workload": w.name, "B": w.B, "H_q": w.H_q, "H_kv": w.H_kv, "L": w.L,
                   "d": w.d_k, "seg_len": w.seg_len, "rule": w.rule,
                   "parallelism": f"sp{world} (one run of whole segments per rank; one "
                                  "all-gather of the runs' state updates)",
                   "l2": "inputs larger than L2; steps timed back to back"},
        "tc_peak_frac_step": (flops / (step_ms / 1000.0)) / (peaks["bf16_tflops"] * 1e12),
        "clocks": clocks.summary(), "e2e": None, "cpu_baseline": None,
    }), flush=True)
    return 0


def decode_bytes_per_segment(w):
    """Algorithmic HBM bytes of decoding one full segment (S steps, pos =
    0..S-1): per KV head the buffer rows 0..pos (keys and values), M and z,
    the new k_t, v_t read and written into the buffer; per query head q_t
    read, out_t written and beta."""
    e = 2 if w.dtype == "bf16" else 4
    d, S = w.d_k, w.seg_len
    rows = S * (S + 1) // 2  # sum over pos of (pos + 1)
    per_kv = rows * 2 * d * e + S * (d * d * 4 + d * 4 + 4 * d * e)
    per_q = S * (2 * d * e + 4)
    return w.B * (w.H_kv * per_kv + w.H_q * per_q)


def run_decode_probe(args, w):
    """Three eager decode calls of the workload's shape at one position (the
    buffers hold N(0,1) rows), for a profiler capture of the decode kernel;
    prints no result line."""
    import torch

    from compressive_memory_transformer_segment_b200 import api

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    st = api.DecodeStream(w.B, w.H_q, w.H_kv, w.d_k, w.seg_len, w.rule, dtype=tdt, device=dev)
    gen = torch.Generator(device=dev).manual_seed(w.seed)
    st.k_buf.normal_(generator=gen)
    st.v_buf.normal_(generator=gen)
    st.z.fill_(1.0)
    q = torch.randn((w.B, w.H_q, w.d_k), generator=gen, device=dev).to(tdt)
    k = torch.randn((w.B, w.H_kv, w.d_k), generator=gen, device=dev).to(tdt)
    v = torch.randn((w.B, w.H_kv, w.d_k), generator=gen, device=dev).to(tdt)
    beta = torch.zeros(w.H_q, device=dev)
    pos = min(max(args.decode_probe, 0), w.seg_len - 2)
    for _ in range(3):
        st.pos = pos
        st.step(q, k, v, beta)
    api.sync_status()
    torch.cuda.synchronize(dev)
    return 0


def run_decode(args, w):
    """Streaming decode: one token per (batch row, head) per call, `steps`
    full segments of the workload's shape (S calls each; the state update
    runs once per segment).  Single GPU."""
    import torch

    from compressive_memory_transformer_segment_b200 import api

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    api.load_library()
    S = w.seg_len
    ws_ = w.with_(L=2 * S)
    inp = synth.make_inputs(ws_)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def dev_tensor(x):
        if w.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dev)

    q, k, v = (dev_tensor(inp[n]) for n in ("q", "k", "v"))
    beta = torch.from_numpy(inp["beta"]).to(dev)
    # A prior state (the memory after the first segment), then the second
    # segment's tokens, each [B, heads, d] contiguous.
    M0, z0 = api.init_state(w.B, w.H_kv, w.d_k, w.d_v, device=dev)
    M0, z0 = api.state_update(k[:, :, :S].contiguous(), v[:, :, :S].contiguous(), M0, z0, S, w.rule)
    qt = q[:, :, S:].permute(2, 0, 1, 3).contiguous()
    kt = k[:, :, S:].permute(2, 0, 1, 3).contiguous()
    vt = v[:, :, S:].permute(2, 0, 1, 3).contiguous()
    st = api.DecodeStream(w.B, w.H_q, w.H_kv, w.d_k, S, w.rule, dtype=tdt, device=dev, M=M0, z=z0)
    out = torch.empty((w.B, w.H_q, w.d_v), dtype=tdt, device=dev)
    stream = torch.cuda.current_stream(dev)

    def segment(strm):
        for t in range(S):
            st.step(qt[t], kt[t], vt[t], beta, out=out, stream=strm)

    for _ in range(args.warmup):
        segment(stream)
    api.sync_status(stream)
    # Eager calls with per-kernel CUDA events: the decode kernels' device time.
    api.set_kernel_timing(True)
    api.kernel_times(reset=True)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    segment(stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    eager_ms = e0.elapsed_time(e1)
    api.set_kernel_timing(False)
    ktimes = api.kernel_times(reset=True)
    api.sync_status(stream)
    # The timed steps: one CUDA graph per segment (its S calls and the state
    # update), replayed, so that host launch overhead is not measured.
    graph, graph_note = torch.cuda.CUDAGraph(), "each timed step replays one CUDA graph of the segment's calls"
    try:
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(graph, stream=cap):
            segment(cap)
        stream.wait_stream(cap)
        run = graph.replay
    except Exception as exc:  # capture refused: time eager calls instead
        torch.cuda.synchronize(dev)
        graph_note = f"graph capture failed ({type(exc).__name__}); eager calls timed"
        st.pos = 0

        def run():
            segment(stream)
    for _ in range(args.warmup):
        run()
    api.sync_status(stream)
    torch.cuda.synchronize(dev)
    with ClockSampler(0) as clocks:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            run()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    elapsed_ms = e0.elapsed_time(e1)
    api.sync_status(stream)
    tokens = w.B * S * args.steps
    value = tokens / (elapsed_ms / 1000.0)

    # End to end: each token's q_t, k_t, v_t copied from pinned host memory
    # and out_t copied back, inside the timed region (one segment).
    hq, hk, hv = (x.cpu().pin_memory() for x in (qt, kt, vt))
    hout = torch.empty((S,) + tuple(out.shape), dtype=tdt).pin_memory()
    dq, dk, dv = torch.empty_like(qt[0]), torch.empty_like(kt[0]), torch.empty_like(vt[0])
    torch.cuda.synchronize(dev)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for t in range(S):
        dq.copy_(hq[t], non_blocking=True)
        dk.copy_(hk[t], non_blocking=True)
        dv.copy_(hv[t], non_blocking=True)
        st.step(dq, dk, dv, beta, out=out, stream=stream)
        hout[t].copy_(out, non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize(dev)
    e2e_value = w.B * S / (e2.elapsed_time(e3) / 1000.0)

    peaks, peak_src = load_peaks()
    dec_ms, dec_n = ktimes["attention"]
    scan_ms, scan_n = ktimes["state_scan"]
    seg_bytes = decode_bytes_per_segment(w)
    # The decode kernels' time inside the timed graph replays: the step minus
    # its one state update (timed with events in the eager pass).
    graph_dec_ms = elapsed_ms / args.steps - scan_ms
    achieved = seg_bytes / (graph_dec_ms / 1000.0) / 1e9
    plan = api.plan(api.make_dims(w.B, w.H_q, w.H_kv, S, w.d_k, w.d_v, tdt), S, w.rule)
    line = {
        "metric": "Infini-attention streaming decode tokens/s on 1 B200 (one token per call)",
        "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "step": f"one segment: {S} decode calls of one token per (batch row, head), "
                "then the segment's state update",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded Philox N(0,1) q/k/v, U(-r,r) beta)",
        "config": {"workload": f"{w.name} decode", "B": w.B, "H_q": w.H_q, "H_kv": w.H_kv,
                   "d": w.d_k, "seg_len": S, "rule": w.rule, "io_dtype": w.dtype,
                   "l2": "buffers and state stay in L2 between calls (as in serving)"},
        "clocks": clocks.summary(),
        "e2e": {"value": e2e_value, "unit": "tokens/s", "note": "eager calls, per-token copies",
                "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in (hq, hk, hv)),
                "d2h_bytes_per_step": hout.numel() * hout.element_size(), "steps": 1},
        # one decode kernel per call, plus the state update's scan kernels
        # once per segment
        "gpu_launches": (S + plan["launches"] - 1) * args.steps,
        "roofline": {"bound": "hbm", "kernel": "decode attention (partial + combine)",
                     "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "peak_source": f"{peak_src} copy",
                     "traffic": None,
                     "algorithmic_bytes_per_step": seg_bytes,
                     "avg_call_us": graph_dec_ms * 1000.0 / S,
                     "eager_avg_call_us": dec_ms * 1000.0 / max(dec_n, 1),
                     "timing": "decode calls inside the timed graph replays (step time minus "
                               "the state update's event-timed duration), per call"},
        "kernel_ms": {"decode_per_segment": dec_ms, "state_update_per_segment": scan_ms},
        "eager_tokens_per_s": w.B * S / (eager_ms / 1000.0),
        "graph": graph_note,
        "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)
    return 0


def backward_flops(w):
    """Algorithmic fp32 flops of the backward kernels (the recompute of the
    states excluded), per step: per (batch row, query head, segment of n
    rows) the attention's six causal n x n x d products (scores and A_dot
    recomputed, dP, dV, dQ, dK: 6 n (n + 1) d) and the retrieval's three
    n x d x d products (A_mem recomputed, dM, d sigma(Q): 6 n d^2); per
    (batch row, KV head, segment) the update's VJP: 2 products (linear) or
    5 (delta) of n x d x d."""
    d = w.d_k
    per_kv = (4 if w.rule == "linear" else 10)
    total = 0
    for s in range(-(-w.L // w.seg_len)):
        n = min(w.seg_len, w.L - s * w.seg_len)
        total += w.B * w.H_q * (6 * n * (n + 1) * d + 6 * n * d * d)
        total += w.B * w.H_kv * per_kv * n * d * d
    return total


def oracle_backward_sample(w, budget_s):
    """Time the float64 oracle's backward on whole (batch row, KV head) chains
    until about ``budget_s`` seconds have passed; token-equivalents/s as in
    oracle_sample."""
    import oracle  # the CPU baseline is the only product-adjacent use of the oracle

    g = w.H_q // w.H_kv
    beta = synth.make_beta(w).astype(np.float64)
    grads = synth.make_output_grads(w)
    one = w.with_(B=1, H_q=g, H_kv=1)
    rows, used, elapsed = 0, [], 0.0
    for b in range(w.B):
        for j in range(w.H_kv):
            kc = synth.as_float64(synth.make_head(w, "k", b, j), w.dtype)[None, None]
            vc = synth.as_float64(synth.make_head(w, "v", b, j), w.dtype)[None, None]
            heads = list(range(j * g, (j + 1) * g))
            qc = np.stack([synth.as_float64(synth.make_head(w, "q", b, h), w.dtype)
                           for h in heads])[None]
            dout = synth.as_float64(grads["dout"][b, heads], w.dtype)[None]
            t0 = time.perf_counter()
            oracle.infini_attention_backward(
                qc, kc, vc, beta[heads], np.zeros((1, 1, w.d_k, w.d_v)), np.zeros((1, 1, w.d_k)),
                w.seg_len, w.rule, dout, grads["dM_out"][b:b + 1, j:j + 1].astype(np.float64),
                grads["dz_out"][b:b + 1, j:j + 1].astype(np.float64))
            elapsed += time.perf_counter() - t0
            rows += w.L
            used.append((b, j))
            if elapsed >= budget_s:
                break
        if elapsed >= budget_s:
            break
    desc = (f"oracle backward (NumPy float64), {len(used)} whole (batch, KV head) chain(s) "
            f"from {used[0]}, each with its {g} query head(s), {one.L} rows each, in "
            f"{elapsed:.2f} s of compute (input generation untimed); token-equivalents = "
            f"rows / H_kv")
    return rows / w.H_kv / elapsed, desc


def run_backward(args, w):
    """The backward through the segments (gradients of every input given the
    gradients of out, M_out, z_out) on one GPU; a step is one
    infini_attn_backward over one batch, from the zero initial memory."""
    import torch

    from compressive_memory_transformer_segment_b200 import api

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    api.load_library()
    inp = synth.make_inputs(w)
    grads = synth.make_output_grads(w)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def host_tensor(x):
        if w.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))

    hq, hk, hv, hd = (host_tensor(a) for a in (inp["q"], inp["k"], inp["v"], grads["dout"]))
    q, k, v, dout = (t.to(dev) for t in (hq, hk, hv, hd))
    beta = torch.from_numpy(inp["beta"]).to(dev)
    M0, z0 = api.init_state(w.B, w.H_kv, w.d_k, w.d_v, device=dev)
    dM = torch.from_numpy(grads["dM_out"]).to(dev)
    dz = torch.from_numpy(grads["dz_out"]).to(dev)
    dims = api.make_dims(w.B, w.H_q, w.H_kv, w.L, w.d_k, w.d_v, tdt)
    nbytes = api.backward_workspace_bytes(dims, w.seg_len, w.rule)
    if nbytes == 0:
        print(json.dumps({"metric": "Infini-attention backward", "unsupported": w.name}))
        return 1
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v, dout))
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if in_bytes < 2 * L2_BYTES else None

    def step():
        return api.backward(q, k, v, beta, M0, z0, w.seg_len, w.rule, dout, dM, dz,
                            workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    api.sync_status(stream)

    def timed_pass(n):
        total = 0.0
        for _ in range(n):
            if flush is not None:
                flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            total += e0.elapsed_time(e1)
        return total

    # Per-kernel times from a separate pass (their events would add gaps).
    api.set_kernel_timing(True)
    api.kernel_times(reset=True)
    timed_pass(args.steps)
    api.set_kernel_timing(False)
    ktimes = api.kernel_times(reset=True)
    torch.cuda.synchronize(dev)
    with ClockSampler(0) as clocks:
        elapsed_ms = timed_pass(args.steps)
    api.sync_status(stream)
    tokens = w.B * w.L * args.steps
    value = tokens / (elapsed_ms / 1000.0)

    # End to end: inputs and upstream gradients copied from pinned host memory,
    # the six gradients copied back, inside the timed region.
    hp = [t.pin_memory() for t in (hq, hk, hv, hd)]
    dev_in = [torch.empty_like(t, device=dev) for t in hp]
    outs_h = None
    e2e_steps = max(1, min(args.steps, 5))
    torch.cuda.synchronize(dev)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(e2e_steps):
        for dst, src in zip(dev_in, hp):
            dst.copy_(src, non_blocking=True)
        res = api.backward(*dev_in[:3], beta, M0, z0, w.seg_len, w.rule, dev_in[3], dM, dz,
                           workspace=ws, stream=stream)
        if outs_h is None:
            outs_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in res]
        for dst, src in zip(outs_h, res):
            dst.copy_(src, non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize(dev)
    e2e_value = w.B * w.L * e2e_steps / (e2.elapsed_time(e3) / 1000.0)

    scan_ms, scan_n = ktimes["state_scan"]
    bwd_ms, bwd_n = ktimes["attention"]
    flops = backward_flops(w)
    sm_mhz = (clocks.summary() or {}).get("sm_max_mhz") or 1965
    fp32_peak = 148 * 128 * 2 * sm_mhz * 1e6 / 1e12  # FMA lanes x 2 flop x max SM clock
    achieved = flops / (bwd_ms / max(bwd_n, 1) / 1000.0) / 1e12
    line = {
        "metric": "Infini-attention backward tokens/s on 1 B200 (gradients through the segments)",
        "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded Philox N(0,1) q/k/v and upstream gradients, U(-r,r) beta)",
        "config": {"workload": f"{w.name} backward", "B": w.B, "H_q": w.H_q, "H_kv": w.H_kv,
                   "L": w.L, "d_k": w.d_k, "d_v": w.d_v, "seg_len": w.seg_len,
                   "rule": w.rule, "io_dtype": w.dtype, "grad_dtype": "f32",
                   "l2": ("L2 flushed (256 MiB write) between timed steps; each step timed alone"
                          if flush is not None else "inputs larger than L2")},
        "clocks": clocks.summary(),
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hp),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in outs_h),
                "steps": e2e_steps},
        "gpu_launches": None,
        "roofline": {"bound": "alu", "kernel": "backward kernels (segment VJPs, reverse scan, gate)",
                     "achieved": achieved, "peak": fp32_peak, "unit": "TFLOP/s",
                     "frac": achieved / fp32_peak,
                     "peak_source": "derived: 148 SMs x 128 fp32 FMA lanes x 2 flop x max SM clock",
                     "traffic": None, "algorithmic_flops_per_step": flops,
                     "avg_launch_ms": bwd_ms / max(bwd_n, 1)},
        "kernel_ms": {"state_recompute": scan_ms / max(scan_n, 1),
                      "backward": bwd_ms / max(bwd_n, 1)},
    }
    plan = api.plan(dims, w.seg_len, w.rule)
    line["gpu_launches"] = (plan["launches"] - 1 + 3) * args.steps
    if args.cpu_baseline:
        v, desc = oracle_backward_sample(w, args.cpu_budget)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": host_cores(),
                                "kind": "oracle", "sample": desc}
    print(json.dumps(line), flush=True)
    return 0


def oracle_projection_sample(w, pin, budget_s):
    """Time the float64 oracle's projection prologue on blocks of 256 token
    rows of batch row 0 until about ``budget_s`` seconds have passed."""
    import oracle  # the CPU baseline is the only product-adjacent use of the oracle

    d = w.d_k
    wf = synth.bf16_bits_to_f32(pin["w"]).astype(np.float64)
    bf = pin["bias"].astype(np.float64)
    c64, s64 = oracle.rope_tables(w.L, d)
    rows, elapsed = 0, 0.0
    while elapsed < budget_s and rows < w.L:
        n = min(256, w.L - rows)
        xr = synth.bf16_bits_to_f32(pin["x"][0:1, rows:rows + n]).astype(np.float64)
        t0 = time.perf_counter()
        oracle.qkv_project_rope(xr, wf, bf, c64[rows:rows + n], s64[rows:rows + n], w.H_q,
                                w.H_kv, d)
        elapsed += time.perf_counter() - t0
        rows += n
    desc = (f"oracle (NumPy float64 matmul + rotation), {rows} token rows of batch row 0 in "
            f"blocks of 256, {elapsed:.2f} s of compute (tables and conversion untimed)")
    return rows / elapsed, desc


def run_projection(args, w):
    """The Q/K/V projection prologue: y = x W^T + bias, rotary embedding of the
    query and key heads, bf16 heads in the attention's layout.  A step is one
    infini_attn_qkv_project over the workload's tokens (d_model = H_q d)."""
    import torch

    from compressive_memory_transformer_segment_b200 import api

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    api.load_library()
    d, H_q, H_kv = w.d_k, w.H_q, w.H_kv
    dm = H_q * d
    n_out = (H_q + 2 * H_kv) * d
    pin = synth.make_projection_inputs(w)

    def host_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    hx = host_bf16(pin["x"])
    x = hx.to(dev)
    W = host_bf16(pin["w"]).to(dev)
    bias = torch.from_numpy(pin["bias"]).to(dev)
    cos, sin = api.rope_tables(w.L, d, device=dev)
    q = torch.empty((w.B, H_q, w.L, d), dtype=torch.bfloat16, device=dev)
    k = torch.empty((w.B, H_kv, w.L, d), dtype=torch.bfloat16, device=dev)
    v = torch.empty((w.B, H_kv, w.L, d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    in_bytes = x.numel() * 2 + W.numel() * 2
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if in_bytes < 2 * L2_BYTES else None

    def step():
        api.qkv_project(x, W, bias, cos, sin, H_q, H_kv, d, q=q, k=k, v=v, stream=stream)

    bias_bf16 = bias.to(torch.bfloat16)

    def torch_step():
        # The unfused library route, for context: cuBLAS GEMM with bias, then
        # the rotation and the head layout in PyTorch ops.
        y = torch.nn.functional.linear(x, W, bias_bf16)
        yq, yk, yv = y.split([H_q * d, H_kv * d, H_kv * d], dim=-1)
        out = []
        for part, H, rot in ((yq, H_q, True), (yk, H_kv, True), (yv, H_kv, False)):
            t = part.view(w.B, w.L, H, d).transpose(1, 2)
            if rot:
                t1, t2 = t[..., : d // 2].float(), t[..., d // 2:].float()
                t = torch.cat([t1 * cos - t2 * sin, t2 * cos + t1 * sin], dim=-1).to(torch.bfloat16)
            out.append(t.contiguous())
        return out

    def timed(fn, n):
        total = 0.0
        for _ in range(n):
            if flush is not None:
                flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            total += e0.elapsed_time(e1)
        return total

    for _ in range(args.warmup):
        step()
        torch_step()
    api.sync_status(stream)
    torch.cuda.synchronize(dev)
    with ClockSampler(0) as clocks:
        elapsed_ms = timed(step, args.steps)
    api.sync_status(stream)
    torch_ms = timed(torch_step, args.steps)
    tokens = w.B * w.L * args.steps
    value = tokens / (elapsed_ms / 1000.0)

    # End to end: x from pinned host memory in, q / k / v back to pinned host
    # memory, inside the timed region (weights and tables stay resident).
    e2e = None
    if args.e2e:
        hxp = hx.pin_memory()
        outs_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (q, k, v)]
        e2e_steps = max(1, min(args.steps, 3))
        torch.cuda.synchronize(dev)
        e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2.record(stream)
        for _ in range(e2e_steps):
            x.copy_(hxp, non_blocking=True)
            step()
            for dst, src in zip(outs_h, (q, k, v)):
                dst.copy_(src, non_blocking=True)
        e3.record(stream)
        torch.cuda.synchronize(dev)
        e2e = {"value": w.B * w.L * e2e_steps / (e2.elapsed_time(e3) / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": hx.numel() * 2,
               "d2h_bytes_per_step": sum(t.numel() * 2 for t in outs_h), "steps": e2e_steps}

    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    flops = 2.0 * w.B * w.L * n_out * dm
    traffic = attention_traffic(w.name, PROJECTION_TRAFFIC)
    achieved = flops / (elapsed_ms / args.steps / 1000.0) / 1e12
    line = {
        "metric": "Q/K/V projection + rotary embedding tokens/s on 1 B200",
        "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Philox N(0,1) x, N(0,1/d_model) weights, N(0,0.01) bias)",
        "config": {"workload": f"{w.name} projection prologue", "B": w.B, "L": w.L,
                   "d_model": dm, "H_q": H_q, "H_kv": H_kv, "d": d, "n_out": n_out,
                   "rope": "rotate-half, base 10000, positions 0..L-1",
                   "l2": ("L2 flushed (256 MiB write) between timed steps; each step timed alone"
                          if flush is not None else "inputs larger than L2")},
        "clocks": clocks.summary(),
        "e2e": e2e,
        "gpu_launches": args.steps,
        "roofline": {"bound": "tensor", "kernel": "qkv_rope", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peak_src} bf16 (burst)",
                     "traffic": traffic["bytes"] if traffic else None,
                     "traffic_note": (f"{traffic['note']}; {traffic['profile']}" if traffic
                                      else "no capture of this kernel source for this workload"),
                     "algorithmic_flops_per_step": flops,
                     "avg_launch_ms": elapsed_ms / args.steps},
        "library_route_ms": torch_ms / args.steps,
    }
    if args.cpu_baseline:
        v_cpu, desc = oracle_projection_sample(w, pin, args.cpu_budget)
        line["cpu_baseline"] = {"value": v_cpu, "unit": "tokens/s", "cores": host_cores(),
                                "kind": "oracle", "sample": desc}
    print(json.dumps(line), flush=True)
    return 0


def run_layer(args, w):
    """The whole layer from its input: the Q/K/V projection prologue with the
    rotary embedding, then the forward (attention, retrieval, gate, memory
    update) on the heads it wrote, both through the C ABI on one stream.  A
    step is one pass over the workload's tokens (d_model = H_q d)."""
    import torch

    from compressive_memory_transformer_segment_b200 import api

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    api.load_library()
    d, H_q, H_kv = w.d_k, w.H_q, w.H_kv
    dm = H_q * d
    n_out = (H_q + 2 * H_kv) * d
    pin = synth.make_projection_inputs(w)

    def host_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    x = host_bf16(pin["x"]).to(dev)
    W = host_bf16(pin["w"]).to(dev)
    bias = torch.from_numpy(pin["bias"]).to(dev)
    cos, sin = api.rope_tables(w.L, d, device=dev)
    q = torch.empty((w.B, H_q, w.L, d), dtype=torch.bfloat16, device=dev)
    k = torch.empty((w.B, H_kv, w.L, d), dtype=torch.bfloat16, device=dev)
    v = torch.empty((w.B, H_kv, w.L, d), dtype=torch.bfloat16, device=dev)
    beta = torch.from_numpy(synth.make_beta(w)).to(dev)
    M0, z0 = api.init_state(w.B, H_kv, d, d, device=dev)
    dims = api.make_dims(w.B, H_q, H_kv, w.L, d, d, torch.bfloat16)
    plan = api.plan(dims, w.seg_len, w.rule)
    ws = torch.empty(plan["workspace_bytes"], dtype=torch.uint8, device=dev)
    out = torch.empty((w.B, H_q, w.L, d), dtype=torch.bfloat16, device=dev)
    M1, z1 = torch.empty_like(M0), torch.empty_like(z0)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if x.numel() * 2 < 2 * L2_BYTES else None

    def step():
        api.qkv_project(x, W, bias, cos, sin, H_q, H_kv, d, q=q, k=k, v=v, stream=stream)
        api.forward(q, k, v, beta, M0, z0, w.seg_len, w.rule, out=out, M_out=M1, z_out=z1,
                    workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    api.sync_status(stream)
    torch.cuda.synchronize(dev)
    total = 0.0
    with ClockSampler(0) as clocks:
        for _ in range(args.steps):
            if flush is not None:
                flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            total += e0.elapsed_time(e1)
    api.sync_status(stream)
    ms = total / args.steps
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    flops = 2.0 * w.B * w.L * n_out * dm + configs.algorithmic_flops(w)
    achieved = flops / (ms / 1000.0) / 1e12
    line = {
        "metric": "Infini-attention layer (Q/K/V projection + rotary embedding + forward) tokens/s "
                  "on 1 B200",
        "value": w.B * w.L / (ms / 1000.0), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Philox N(0,1) x, N(0,1/d_model) weights, U(-r,r) beta)",
        "config": {"workload": f"{w.name} layer", "B": w.B, "L": w.L, "d_model": dm, "H_q": H_q,
                   "H_kv": H_kv, "d": d, "seg_len": w.seg_len, "rule": w.rule,
                   "l2": ("L2 flushed (256 MiB write) between timed steps"
                          if flush is not None else "inputs larger than L2")},
        "clocks": clocks.summary(),
        "e2e": None,
        "gpu_launches": (1 + plan["launches"]) * args.steps,
        "roofline": {"bound": "tensor", "kernel": "whole layer (projection GEMM + attention + scan)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peak_src} bf16 (burst)", "traffic": None,
                     "algorithmic_flops_per_step": flops},
        "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(configs.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false",
                    help="skip the host-buffer end-to-end measurement (profiling runs)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size (smaller profiling captures)")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override the workload's sequence length L (smaller profiling captures)")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline sample")
    ap.add_argument("--reference-budget", type=float, default=60.0,
                    help="total seconds of oracle work for --impl reference")
    ap.add_argument("--decode-probe", type=int, default=None, metavar="POS",
                    help="three eager decode calls at position POS, no result line "
                         "(for a profiler capture of the decode kernel)")
    ap.add_argument("--shard", choices=["replicas", "chains"], default="replicas",
                    help="replicas: every rank runs the whole workload (weak scaling); chains: "
                         "the workload's (batch row, KV head) chains are split, one block per "
                         "rank (strong scaling)")
    ap.add_argument("--seq-parallel", action="store_true",
                    help="sequence-parallel linear rule over the ranks (strong scaling)")
    ap.add_argument("--backward", action="store_true",
                    help="the backward through the segments (gradients of every input); "
                         "short-segment shapes (seg_len <= 64, d in {32, 64})")
    ap.add_argument("--decode", action="store_true",
                    help="streaming decode (one token per call) of the workload's shape; "
                         "a step is one full segment")
    ap.add_argument("--projection", action="store_true",
                    help="the Q/K/V projection + rotary embedding prologue of the workload's "
                         "shape (d_model = H_q d)")
    ap.add_argument("--layer", action="store_true",
                    help="the whole layer from its input: the projection prologue, then the "
                         "forward on the heads it wrote")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    w = configs.WORKLOADS[args.config]
    if args.batch is not None:
        w = w.with_(B=args.batch, name=f"{w.name}-B{args.batch}")
    if args.seq_len is not None:
        if args.seq_len <= 0:
            ap.error("--seq-len must be positive")
        w = w.with_(L=args.seq_len, name=f"{w.name}-L{args.seq_len}")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.decode_probe is not None:
        return run_decode_probe(args, w)
    if args.decode:
        return run_decode(args, w)
    if args.backward:
        return run_backward(args, w)
    if args.projection:
        return run_projection(args, w)
    if args.layer:
        return run_layer(args, w)
    if args.seq_parallel:
        return run_seq_parallel(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
