"""Benchmark: varlen causal MLA prefill on B200 through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one ``mla_prefill`` call (plan kernel + attention kernel) over the
whole workload, inputs resident in HBM.  Prints ONE JSON line (rank 0).

* value: algorithmic TFLOP/s = causally visible (query, key, head) triples x 640
  FLOPs (2*192 for Q.K^T plus 2*128 for P.V) / device time per step, summed over
  ranks (each rank runs an independent replica: "scaling": "weak").
* roofline: the attention kernel alone (timed with CUDA events recorded by the
  library around its launch, in a second pass of the same steps) against the
  measured dense bf16 peak; the same launch's algorithmic bytes against the
  measured HBM bandwidth beside it.
* warm_l2: workloads smaller than twice the L2 are timed with the L2 flushed
  before every step; the same steps without the flush are reported here.
* e2e: the same metric through the public call with pinned HOST inputs: every
  step copies the inputs host->device, runs the call and copies attenOut back.
* cpu_baseline: the fp64 CPU oracle on a bounded sample of the same workload.
* --impl reference: the fp64 CPU oracle as the reference arm (rank 0 only).
"""
import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FLOPS_PER_TRIPLE = 640  # 2*(128+64) for the two-part Q.K^T, 2*128 for P.V
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def visible_triples(wl):
    """Causally visible (query, key) pairs over all sequences, times the head count."""
    n = 0
    for lq, lk in zip(wl.q_seqlens, wl.kv_seqlens):
        per_row = np.clip(np.arange(lq) + (lk - lq) + 1, 0, lk) if wl.causal else np.full(lq, lk)
        n += int(per_row.sum())
    return n * wl.head_num


def algorithmic_bytes(wl):
    """Read Q, Q_rope, K, K_rope, V once and write O once (16-bit elements)."""
    return 2 * (wl.t_q * wl.head_num * (wl.d_nope + wl.d_rope) + wl.t_k * wl.kv_head_num * (
        wl.d_nope + wl.d_rope + wl.d_nope) + wl.t_q * wl.head_num * wl.d_nope)


KERNEL_SOURCES = ["mla_prefill_attention_varlen_b200/csrc/mla_prefill_sm100.cuh",
                  "mla_prefill_attention_varlen_b200/csrc/mla_prefill_pair_sm100.cuh",
                  "mla_prefill_attention_varlen_b200/csrc/sm100_ptx.cuh"]
# the fused MLA Prolog q kernel (its traffic entry in profiles/traffic.json is keyed on these)
PROLOG_Q_SOURCES = ["mla_prefill_attention_varlen_b200/csrc/prolog_q_sm100.cuh",
                    "mla_prefill_attention_varlen_b200/csrc/mla_prefill_sm100.cuh",
                    "mla_prefill_attention_varlen_b200/csrc/sm100_ptx.cuh"]


def kernel_sources_hash(sources=None):
    """sha256 over the device-code sources (a measured traffic figure is only valid for this code)."""
    import hashlib

    h = hashlib.sha256()
    for rel in sources or KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# attention kernel of a prefill call (mla_prefill_last_kernel) -> its name
KERNEL_NAMES = {1: "mla_prefill_sm100_kernel", 2: "mla_prefill_pair_kernel"}


def measured_traffic(workload, sources=None):
    """DRAM bytes per launch from the committed ncu figures (profiles/traffic.json), or None when
    there is no figure for this workload or it was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        entry = json.load(f).get("launches", {}).get(workload)
    if not entry or entry.get("kernel_sources_sha256") != kernel_sources_hash(sources):
        return None
    try:
        return int(entry["traffic_bytes_per_launch"])
    except (KeyError, TypeError, ValueError):
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) samples taken while the timed region runs.

    Samples come from NVML every ~20 ms in a background thread, stamped with the
    host clock; only samples inside [mark_start, mark_stop] are summarised.  The
    GPU is found by its UUID (CUDA and NVML may number devices differently).
    Falls back to `nvidia-smi -lms 100` when NVML is unavailable.
    """

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index, period=0.02):
        self.cuda_index = cuda_index
        self.period = period
        self.samples = []
        self.t0 = self.t1 = None
        self._stop = False
        self._thread = None
        self._proc = None
        self.source = None

    def _uuid(self):
        import torch

        try:
            u = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            return None

    def __enter__(self):
        import threading

        uuid = self._uuid()
        try:
            import pynvml

            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid else pynvml.nvmlDeviceGetHandleByIndex(0)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons", None))

            def loop():
                while not self._stop:
                    t = time.perf_counter()
                    try:
                        self.samples.append((t, pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                             pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM),
                                             int(get_reasons(h))))
                    except Exception:
                        pass
                    time.sleep(self.period)

            self._thread = threading.Thread(target=loop, daemon=True)
            self._thread.start()
            self.source = "nvml"
        except Exception:
            self.source = "nvidia-smi"
            sel = ["-i", uuid] if uuid else []
            try:
                self._proc = subprocess.Popen(
                    ["nvidia-smi"] + sel + ["--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                                            "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self._proc_t0 = time.perf_counter()
            except (OSError, ValueError):
                self._proc = None
        return self

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_stop(self):
        self.t1 = time.perf_counter()

    def __exit__(self, *exc):
        self._stop = True
        if self._thread is not None:
            self._thread.join(1.0)
        if self._proc is not None:
            self._proc.terminate()
            try:
                out, _ = self._proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
                out, _ = self._proc.communicate()
            # nvidia-smi lines carry no host stamps: spread them evenly over the process lifetime
            lines = [l for l in (out or "").strip().splitlines() if l.count(",") >= 2]
            t_end = time.perf_counter()
            for k, line in enumerate(lines):
                parts = [x.strip() for x in line.split(",")]
                try:
                    t = self._proc_t0 + (t_end - self._proc_t0) * (k + 0.5) / max(1, len(lines))
                    self.samples.append((t, float(parts[0]), float(parts[1]), int(parts[2], 16)))
                except ValueError:
                    continue

    def summary(self):
        inside = [s for s in self.samples if self.t0 is None or (self.t0 <= s[0] <= (self.t1 or s[0]))]
        if not inside:
            inside = self.samples
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        reasons = set()
        for s in inside:
            for bit, name in self.REASONS.items():
                if s[3] & bit:
                    reasons.add(name)
        return {"sm_mhz": float(np.median([s[1] for s in inside])), "sm_max_mhz": float(max(s[2] for s in inside)),
                "reasons": sorted(reasons), "samples": len(inside), "source": self.source}


def dist_setup(n_gpus):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world):
    """The maximum of a per-rank float over all ranks (device time is that of the slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank, ms_max):
    """Whole-job rate: every rank processes units_per_rank in (at most) ms_max milliseconds."""
    return world * units_per_rank / (ms_max * 1e-3)


def time_oracle_sample(wl, x_cpu, target_s, seed=0):
    """Runs the CPU oracle on seeded sample rows (every head) for about target_s seconds.

    Returns (seconds, triples_computed, description)."""
    import oracle

    rng = np.random.default_rng(seed)
    starts = np.concatenate([[0], np.cumsum(wl.q_seqlens)])

    def rows_triples(rows):
        tot = 0
        for t in rows:
            b = int(np.searchsorted(starts, t, side="right") - 1)
            lq, lk = wl.q_seqlens[b], wl.kv_seqlens[b]
            i = t - starts[b]
            tot += int(min(lk, max(0, i + lk - lq + 1))) if wl.causal else lk
        return tot * wl.head_num

    def run(rows):
        t0 = time.perf_counter()
        oracle.prefill(x_cpu["q"], x_cpu["q_rope"], x_cpu["k"], x_cpu["k_rope"], x_cpu["v"], x_cpu["q_seqlen"],
                       x_cpu["kv_seqlen"], wl.head_num, wl.kv_head_num, wl.qk_scale, rows=rows)
        return time.perf_counter() - t0

    rows = np.sort(rng.choice(wl.t_q, size=min(4, wl.t_q), replace=False))
    dt = run(rows)
    rate = rows_triples(rows) / max(dt, 1e-6)  # triples per second
    want_triples = rate * target_s
    avg = max(1.0, rows_triples(np.arange(wl.t_q)) / wl.t_q)
    n = int(min(wl.t_q, max(4, want_triples / avg)))
    rows = np.sort(rng.choice(wl.t_q, size=n, replace=False))
    dt = run(rows)
    trip = rows_triples(rows)
    desc = "%d seeded query rows x %d heads of workload %s (%d visible triples)" % (n, wl.head_num, wl.name, trip)
    return dt, trip, desc


def to_numpy_f64(x):
    return {k: (v.double().numpy() if v.is_floating_point() else v.numpy()) for k, v in x.items()}


METRIC = "causal MLA prefill TFLOP/s (visible pairs x 640 FLOPs), % of B200 dense bf16 peak, tokens/s"


def workload_config(wl):
    """The workload fields both arms report in `config`."""
    return {"workload": wl.name, "description": wl.description, "batch": wl.batch, "t_q": wl.t_q, "t_k": wl.t_k,
            "head_num": wl.head_num, "kv_head_num": wl.kv_head_num, "qk_scale": wl.qk_scale, "mask": "causal",
            "visible_triples": visible_triples(wl)}


def reference_arm(args, wl):
    """The fp64 CPU oracle timed as the reference implementation (rank 0 only)."""
    import torch

    from mla_prefill_attention_varlen_b200 import workloads as W

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    x = to_numpy_f64(W.make_inputs(wl, device="cpu"))
    import oracle

    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        time_oracle_sample(wl, x, min(per_step, 2.0), seed=1)
    times, trips, desc = [], [], ""
    for k in range(args.steps):
        dt, tr, desc = time_oracle_sample(wl, x, per_step, seed=10 + k)
        times.append(dt)
        trips.append(tr)
    tflops = sum(trips) * FLOPS_PER_TRIPLE / sum(times) / 1e12
    line = {
        "impl": "reference", "metric": METRIC,
        "value": tflops, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(wl), sampled="oracle on seeded query rows of every sequence and head"),
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": oracle.core_count(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def paged_inputs(wl, block_size, device, seed=7):
    """A paged K/V cache holding the workload's keys: K rows [nope | rope] (192), V rows (128),
    blocks assigned to the sequences in a seeded random order (a fragmented cache)."""
    from mla_prefill_attention_varlen_b200 import workloads as W

    x = W.make_inputs(wl, device=device)
    kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], wl.kv_seqlens, block_size, seed=seed)
    return kc, vc, table, x["kv_seqlen"]


def bench_paged(args):
    """mla_paged_cache_load on the cached prefix of a workload: GB/s of bytes read + written."""
    import torch

    import mla_prefill_attention_varlen_b200 as mla
    from mla_prefill_attention_varlen_b200 import workloads as W

    rank, world, local = dist_setup(args.gpus)
    wl = W.get(args.workload)
    dev = torch.device("cuda", torch.cuda.current_device())
    mla.load_library()
    kc, vc, table, lens = paged_inputs(wl, args.block_size, dev)
    T, G = wl.t_k, wl.kv_head_num
    key = torch.empty(T, G, kc.shape[3], dtype=kc.dtype, device=dev)
    value = torch.empty(T, G, vc.shape[3], dtype=vc.dtype, device=dev)
    moved = 2 * (key.numel() + value.numel()) * key.element_size()  # each byte read once and written once
    stream = torch.cuda.current_stream()

    def step():
        mla.mla_paged_cache_load(kc, vc, table, lens, key, value, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    smi = ClockSampler(torch.cuda.current_device())
    barrier(world)
    with smi:
        time.sleep(0.1)
        smi.mark_start()
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            stops[i].record(stream)
        torch.cuda.synchronize()
        smi.mark_stop()
    barrier(world)
    ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in zip(starts, stops)])), world)
    st = mla.mla_prefill_device_status()
    if st != 0:
        raise RuntimeError("device status: %s" % mla.mla_status_string(st))
    gbs = job_throughput(world, moved, ms) / 1e9
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    line = {
        "metric": "paged KV-cache gather GB/s (bytes read + written)", "value": gbs, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16" if kc.dtype == torch.float16 else "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name + "_paged_prefix", "tokens": T, "kv_heads": G, "key_dim": kc.shape[3],
                   "value_dim": vc.shape[3], "block_size": args.block_size, "blocks": kc.shape[0],
                   "l2": "cache %.2f GB > 126 MB L2" % (moved / 2e9)},
        "roofline": {"bound": "hbm", "achieved": gbs / world, "peak": peak, "unit": "GB/s",
                     "frac": gbs / world / peak, "traffic": None, "peak_source": peak_src,
                     "kernel": "paged_gather_kernel", "algorithmic_bytes_per_launch": moved},
        "gpu_launches": 2 * args.steps, "clocks": smi.summary(), "cpu_baseline": None, "e2e": None,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def bench_prolog(args):
    """mla_prolog on the page's configuration: projection TFLOP/s for the whole step, plus the
    HBM roofline of the per-head RmsNorm / RoPE kernel (the largest kernel of this library in it)."""
    import torch

    import mla_prefill_attention_varlen_b200 as mla
    from mla_prefill_attention_varlen_b200 import workloads as W

    rank, world, local = dist_setup(args.gpus)
    s = W.prolog_shapes()["prolog"]
    if args.tokens:
        s.tokens = args.tokens
    dev = torch.device("cuda", torch.cuda.current_device())
    mla.load_library()
    x = W.make_prolog_inputs(s, device=dev)
    order = ("token_x", "wq_a", "wq_b", "wkv", "rope_cos", "rope_sin", "gamma_cq", "gamma_ckv")
    t, h, r, H, d, R = s.tokens, s.hidden, s.q_lora_rank, s.num_heads, s.head_dim, s.rope_dim
    q = torch.empty(t, H, d, dtype=torch.bfloat16, device=dev)
    kv = torch.empty(t, d, dtype=torch.bfloat16, device=dev)
    cq = torch.empty(t, r, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def call(inp, qo, kvo, cqo):
        mla.mla_prolog(*[inp[k] for k in order], H, qo, kvo, cqo, stream=stream)

    flops = 2.0 * t * (h * r + r * H * d + h * d)
    q_flops = 2.0 * t * r * H * d  # the q projection (the fused kernel's work)
    norm_bytes = t * H * d * (4 + 2) + 2 * t * R * 2  # fp32 rows in, bf16 rows out, cos / sin
    q_bytes = 2 * (t * r + r * H * d + t * H * d + 2 * t * R)  # c^Q, wq_b, q, cos / sin once
    mla.set_prolog_path(args.prolog_path)
    for _ in range(args.warmup):
        call(x, q, kv, cq)
    torch.cuda.synchronize()
    fused = mla.prolog_last_fused()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    k_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    k_stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    smi = ClockSampler(torch.cuda.current_device())
    barrier(world)
    with smi:
        time.sleep(0.1)
        smi.mark_start()
        for i in range(args.steps):
            mla.set_profile_events(k_starts[i], k_stops[i])
            starts[i].record(stream)
            call(x, q, kv, cq)
            stops[i].record(stream)
        mla.set_profile_events(None, None)
        torch.cuda.synchronize()
        smi.mark_stop()
    barrier(world)
    ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in zip(starts, stops)])), world)
    kms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in zip(k_starts, k_stops)])), world)
    value = job_throughput(world, flops, ms) / 1e12
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    in_bytes = sum(v.numel() * v.element_size() for v in x.values())

    e2e = None
    if not args.no_e2e:
        hx = {k: v.cpu().pin_memory() for k, v in x.items()}
        dx = {k: torch.empty_like(v) for k, v in x.items()}
        hq = torch.empty(q.shape, dtype=q.dtype).pin_memory()
        hkv = torch.empty(kv.shape, dtype=kv.dtype).pin_memory()

        def e2e_step():
            for k in dx:
                dx[k].copy_(hx[k], non_blocking=True)
            call(dx, q, kv, None)
            hq.copy_(q, non_blocking=True)
            hkv.copy_(kv, non_blocking=True)

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 10))
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world)
        e2e = {"value": world * flops / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": int(in_bytes),
               "d2h_bytes_per_step": int(hq.numel() * 2 + hkv.numel() * 2)}

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle.prolog as prolog

        cpu = {k: v.cpu() for k, v in x.items()}
        n = 8
        t0 = time.time()
        reps = 0
        while True:
            sub = dict(cpu, token_x=cpu["token_x"][:n], rope_cos=cpu["rope_cos"][:n], rope_sin=cpu["rope_sin"][:n])
            prolog.mla_prolog(*[sub[k] for k in order], H)
            reps += 1
            if time.time() - t0 > min(args.cpu_seconds, 10.0):
                break
        dt = time.time() - t0
        cpu_baseline = {"value": reps * n * flops / t / dt / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(),
                        "kind": "oracle", "sample": "%d x %d tokens of the prolog workload (fp64 numpy)" % (reps, n)}

    line = {
        "metric": "MLA prolog TFLOP/s (projection FLOPs 2 t (h r + r H d + h d))", "value": value,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "prolog", "tokens": t, "hidden": h, "q_lora_rank": r, "num_heads": H, "head_dim": d,
                   "rope_dim": R, "weights": "random init", "l2": "inputs and outputs %.2f GB > 126 MB L2" % (
                       (in_bytes + q.numel() * 2) / 1e9),
                   "q_path": "fused tcgen05 q kernel" if fused else "library GEMM + row kernel"},
        "roofline": ({"bound": "tensor", "achieved": q_flops / (kms * 1e-3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                      "frac": q_flops / (kms * 1e-3) / 1e12 / peak,
                      "traffic": measured_traffic("prolog_q_%d" % t, PROLOG_Q_SOURCES), "peak_source": peak_src,
                      "kernel": "mla_prolog_q_kernel (q projection + per-head RmsNorm + RoPE)", "kernel_ms": kms,
                      "algorithmic_flops_per_launch": q_flops, "algorithmic_bytes_per_launch": q_bytes,
                      "hbm_achieved_gbs": q_bytes / (kms * 1e-3) / 1e9, "step_tensor_frac": value / world / peak}
                     if fused else
                     {"bound": "hbm", "achieved": norm_bytes / (kms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                      "frac": norm_bytes / (kms * 1e-3) / 1e9 / hbm, "traffic": None, "peak_source": peak_src,
                      "kernel": "rms_norm_rope_kernel (q rows)", "kernel_ms": kms,
                      "algorithmic_bytes_per_launch": norm_bytes,
                      "step_tensor_frac": value / world / peak}),
        "cpu_baseline": cpu_baseline, "e2e": e2e, "gpu_launches": 2 * args.steps, "clocks": smi.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def time_other_config(name, steps, warmup, peaks):
    """One more workload timed in the same run: step and kernel time (CUDA events), TFLOP/s, the
    kernel's fraction of the measured bf16 peak and, from the same launch, algorithmic bytes per
    kernel time against the measured HBM bandwidth; its own clock samples.  Workloads smaller than
    twice the L2 are timed with the L2 flushed before every step."""
    import torch

    import mla_prefill_attention_varlen_b200 as mla
    from mla_prefill_attention_varlen_b200 import workloads as W

    wl = W.get(name)
    dev = torch.device("cuda", torch.cuda.current_device())
    x = W.make_inputs(wl, device=dev)
    out = torch.empty(wl.t_q, wl.head_num, wl.d_nope, dtype=wl.dtype, device=dev)
    stream = torch.cuda.current_stream()
    in_bytes = sum(t.numel() * t.element_size() for t in x.values())
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev) if in_bytes < 2 * L2_BYTES else None

    def step():
        mla.mla_prefill(x["q"], x["q_rope"], x["k"], x["k_rope"], x["v"], x["q_seqlen"], x["kv_seqlen"],
                        mla.MLA_MASK_CAUSAL, wl.head_num, wl.kv_head_num, wl.qk_scale, out, stream)

    for _ in range(warmup):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(steps)] for _ in range(4)]
    smi = ClockSampler(torch.cuda.current_device())
    with smi:
        time.sleep(0.05)
        smi.mark_start()
        for i in range(steps):  # as a caller's calls run
            if flush is not None:
                flush.zero_()
            ev[0][i].record(stream)
            step()
            ev[1][i].record(stream)
        for i in range(steps):  # events around the attention kernel alone
            if flush is not None:
                flush.zero_()
            mla.set_profile_events(ev[2][i], ev[3][i])
            step()
        mla.set_profile_events(None, None)
        torch.cuda.synchronize()
        smi.mark_stop()
    st = mla.mla_prefill_device_status()
    if st != 0:
        raise RuntimeError("device status after %s: %s" % (name, mla.mla_status_string(st)))
    ms = float(np.mean([a.elapsed_time(b) for a, b in zip(ev[0], ev[1])]))
    kms = float(np.mean([a.elapsed_time(b) for a, b in zip(ev[2], ev[3])]))
    kernel_name = KERNEL_NAMES.get(mla.load_library().mla_prefill_last_kernel(), "none")
    flops = visible_triples(wl) * FLOPS_PER_TRIPLE
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    ab = algorithmic_bytes(wl)
    return {"value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms, "kernel": kernel_name,
            "kernel_ms": kms,
            "kernel_tflops": flops / (kms * 1e-3) / 1e12, "frac": flops / (kms * 1e-3) / 1e12 / peak,
            "hbm_gbs": ab / (kms * 1e-3) / 1e9, "hbm_frac": ab / (kms * 1e-3) / 1e9 / hbm,
            "tokens_per_s": wl.t_q / (ms * 1e-3), "steps": steps, "warmup": warmup,
            "l2": "flushed between steps (512 MB write)" if flush is not None else "inputs %.2f GB > 126 MB L2" % (
                in_bytes / 1e9),
            "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f16", "description": wl.description,
            "clocks": smi.summary()}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--op", default="prefill", choices=["prefill", "prefill_paged", "paged_cache_load", "prolog"],
                    help="prefill: mla_prefill on packed K/V; prefill_paged: mla_prefill_paged reading a "
                         "paged cache in place; paged_cache_load: the gather alone")
    ap.add_argument("--block-size", type=int, default=64, help="paged ops: tokens per cache block")
    ap.add_argument("--tokens", type=int, default=0, help="prolog: tokens (default: the prolog workload's)")
    ap.add_argument("--split", type=int, default=-1,
                    help="split-KV chunk in 128-key tiles for the prefill ops: -1 automatic (default), 0 off")
    ap.add_argument("--other-configs", default="varlen_gqa,chunked,uniform",
                    help="prefill on the default workload: more workloads timed in the same run and reported "
                         "under other_configs (comma-separated; empty for none)")
    ap.add_argument("--prolog-path", type=int, default=-1, choices=[-1, 0],
                    help="prolog: q projection -1 fused kernel where the sizes allow (default), 0 library GEMM")
    ap.add_argument("--kernel", type=int, default=-1, choices=[-1, 1, 2],
                    help="attention kernel: -1 automatic (default), 1 single-CTA, 2 CTA pair")
    ap.add_argument("--heads", type=int, default=0,
                    help="profiling aid: scale head_num and kv_head_num down to this many query heads")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from mla_prefill_attention_varlen_b200 import workloads as W

    wl = W.get(args.workload)
    if args.heads:
        g = wl.head_num // wl.kv_head_num
        wl.head_num, wl.kv_head_num = args.heads, max(1, args.heads // g)
        wl.name += "_h%d" % args.heads
    if args.impl == "reference":
        return reference_arm(args, wl)
    if args.op == "paged_cache_load":
        return bench_paged(args)
    if args.op == "prolog":
        return bench_prolog(args)

    import torch

    import mla_prefill_attention_varlen_b200 as mla

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    mla.load_library()
    mla.set_split_tiles(args.split)
    mla.set_kernel(args.kernel)
    x = W.make_inputs(wl, device=dev)
    out = torch.empty(wl.t_q, wl.head_num, wl.d_nope, dtype=wl.dtype, device=dev)
    H, G, scale = wl.head_num, wl.kv_head_num, wl.qk_scale
    stream = torch.cuda.current_stream()
    paged = args.op == "prefill_paged"
    packed_x = x
    if paged:
        kc, vc, table = W.paged_cache(x["k"], x["k_rope"], x["v"], wl.kv_seqlens, args.block_size, seed=7)
        x = {"q": x["q"], "q_rope": x["q_rope"], "key_cache": kc, "value_cache": vc, "block_tables": table,
             "q_seqlen": x["q_seqlen"], "kv_seqlen": x["kv_seqlen"]}

    def call(d, o):
        if paged:
            mla.mla_prefill_paged(d["q"], d["q_rope"], d["key_cache"], d["value_cache"], d["block_tables"],
                                  d["q_seqlen"], d["kv_seqlen"], mla.MLA_MASK_CAUSAL, H, G, scale, o, stream)
        else:
            mla.mla_prefill(d["q"], d["q_rope"], d["k"], d["k_rope"], d["v"], d["q_seqlen"], d["kv_seqlen"],
                            mla.MLA_MASK_CAUSAL, H, G, scale, o, stream)

    def step(o=out):
        call(x, o)

    in_bytes = sum(t.numel() * t.element_size() for t in x.values())
    flush = None
    if in_bytes < 2 * L2_BYTES:
        flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    st = mla.mla_prefill_device_status()
    if st != 0:
        raise RuntimeError("device status after warm-up: %s" % mla.mla_status_string(st))

    # The K timed steps run exactly as a caller's calls do (no timing hook, so the attention kernel
    # starts while the plan kernel runs); a second pass of K steps records events around the
    # attention kernel alone (hook on) for the roofline.  Clocks are sampled over both.
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    k_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    k_stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    smi = ClockSampler(torch.cuda.current_device())
    torch.cuda.synchronize()
    barrier(world)
    with smi:
        time.sleep(0.1)
        smi.mark_start()
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            starts[i].record(stream)
            step()
            stops[i].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            mla.set_profile_events(k_starts[i], k_stops[i])
            step()
        mla.set_profile_events(None, None)
        torch.cuda.synchronize()
        smi.mark_stop()
    barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, stops)]
    kern_ms = [a.elapsed_time(b) for a, b in zip(k_starts, k_stops)]
    ms = max_over_ranks(float(np.mean(step_ms)), world)
    kms = max_over_ranks(float(np.mean(kern_ms)), world)
    launches_per_step = mla.load_library().mla_prefill_last_launches()  # plan + attention (+ combine)
    kernel_name = KERNEL_NAMES.get(mla.load_library().mla_prefill_last_kernel(), "none")
    st = mla.mla_prefill_device_status()
    if st != 0:
        raise RuntimeError("device status after timing: %s" % mla.mla_status_string(st))

    # Small workloads are timed with a cold L2 (flushed before every step); the same steps with the
    # inputs left in L2 are reported beside them, outside the timed region above.
    warm_ms = warm_kms = None
    if flush is not None:
        w_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        w_stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        wk_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        wk_stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        step()
        for i in range(args.steps):
            mla.set_profile_events(wk_starts[i], wk_stops[i])
            w_starts[i].record(stream)
            step()
            w_stops[i].record(stream)
        mla.set_profile_events(None, None)
        torch.cuda.synchronize()
        warm_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in zip(w_starts, w_stops)])), world)
        warm_kms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in zip(wk_starts, wk_stops)])), world)

    triples = visible_triples(wl)
    flops = triples * FLOPS_PER_TRIPLE
    value = job_throughput(world, flops, ms) / 1e12
    tokens_per_s = job_throughput(world, wl.t_q, ms)
    peaks, peak_src = load_peaks()
    kern_tflops = flops / (kms * 1e-3) / 1e12

    # End to end through the public call: every step copies its inputs from pinned host memory and
    # reads attenOut back.  As a serving pipeline would, step i's host-to-device copy, step i-1's
    # attention and step i-2's device-to-host copy run on three streams, with two device buffers.
    e2e = None
    if not args.no_e2e:
        hx = {k: v.cpu().pin_memory() for k, v in x.items()}
        dx = [{k: torch.empty_like(v) for k, v in x.items()} for _ in range(2)]
        dout = [torch.empty_like(out) for _ in range(2)]
        hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in hx.values())
        d2h = hout[0].numel() * hout[0].element_size()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("in_ready", "in_free", "out_ready", "out_free")}
        for name in ev:
            for e in ev[name]:
                e.record(stream)

        def e2e_step(i):
            b = i % 2
            s_in.wait_event(ev["in_free"][b])
            with torch.cuda.stream(s_in):
                for k in hx:
                    dx[b][k].copy_(hx[k], non_blocking=True)
            ev["in_ready"][b].record(s_in)
            stream.wait_event(ev["in_ready"][b])
            stream.wait_event(ev["out_free"][b])
            call(dx[b], dout[b])
            ev["in_free"][b].record(stream)
            ev["out_ready"][b].record(stream)
            s_out.wait_event(ev["out_ready"][b])
            with torch.cuda.stream(s_out):
                hout[b].copy_(dout[b], non_blocking=True)
            ev["out_free"][b].record(s_out)

        for i in range(args.warmup):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(world)
        e_start = torch.cuda.Event(enable_timing=True)
        e_stop = torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 10))
        e_start.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        stream.wait_stream(s_out)
        e_stop.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e_ms = max_over_ranks(e_start.elapsed_time(e_stop) / n_e2e, world)
        st = mla.mla_prefill_device_status()
        if st != 0:
            raise RuntimeError("device status after the end-to-end steps: %s" % mla.mla_status_string(st))
        e2e = {"value": world * flops / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "pipelined": "h2d / attention / d2h of consecutive steps overlap on three streams"}

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        xc = to_numpy_f64({k: v.cpu() for k, v in packed_x.items()})
        dt, trip, desc = time_oracle_sample(wl, xc, args.cpu_seconds)
        cpu_baseline = {"value": trip * FLOPS_PER_TRIPLE / dt / 1e12, "unit": "TFLOP/s",
                        "cores": oracle.core_count(), "kind": "oracle", "sample": desc}

    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    algo_bytes = algorithmic_bytes(wl)
    # the other workloads, each timed in this run (single GPU, packed K/V, default workload only)
    other = None
    if (world == 1 and not paged and not args.heads and args.split < 0 and args.workload == "long"
            and args.other_configs and args.kernel < 0):
        other = {n: time_other_config(n, args.steps, args.warmup, peaks)
                 for n in args.other_configs.split(",") if n and n != wl.name}
    clocks = smi.summary()
    line = {
        "metric": METRIC + (" (K/V read in place from a paged cache)" if paged else ""),
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f16", "data": "synthetic",
        "config": {**workload_config(wl),
                   "parallelism": "replicas" if world > 1 else "single", "l2": (
                       "flushed between steps (512 MB write)" if flush is not None else
                       "inputs %.2f GB > 126 MB L2" % (in_bytes / 1e9)),
                   "visible_triples": triples, "split_kv": "automatic" if args.split < 0 else args.split,
                   "kernel": {-1: "automatic", 1: "single-CTA", 2: "CTA pair"}[args.kernel],
                   **({"kv_layout": "paged", "block_size": args.block_size, "blocks": int(x["key_cache"].shape[0])}
                      if paged else {"kv_layout": "packed"})},
        "pct_of_peak": 100.0 * value / world / peak,
        "tokens_per_s": tokens_per_s,
        "tflops_counting_1280_flops_per_pair": 2 * value,
        "roofline": {"bound": "tensor", "achieved": kern_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": kern_tflops / peak,
                     "traffic": measured_traffic("%s_paged%d" % (wl.name, args.block_size) if paged else wl.name),
                     "peak_source": peak_src,
                     "peak_kind": "burst", "frac_of_sustained": kern_tflops / peak_sus,
                     "kernel": kernel_name, "kernel_ms": kms,
                     "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": algo_bytes,
                     # the same launch against the HBM roofline (the bound near the ridge, e.g. `uniform`)
                     "hbm_achieved_gbs": algo_bytes / (kms * 1e-3) / 1e9, "hbm_peak_gbs": hbm_peak,
                     "hbm_frac": algo_bytes / (kms * 1e-3) / 1e9 / hbm_peak},
        "warm_l2": None if warm_ms is None else {
            "ms_per_step": warm_ms, "value": job_throughput(world, flops, warm_ms) / 1e12, "unit": "TFLOP/s",
            "kernel_ms": warm_kms, "kernel_frac": flops / (warm_kms * 1e-3) / 1e12 / peak},
        "cpu_baseline": cpu_baseline,
        "e2e": e2e,
        "other_configs": other,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
