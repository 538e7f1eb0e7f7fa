"""Benchmark of the DSA layer on B200: query tokens / second and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|decode|chunked] [--no-extras] [--profile-once]

A step is one pass of the whole hot path over one batch: dsa_layer_forward
(indexer scores -> top-k -> sparse MLA attend) on the workload's synthetic
inputs, already resident in HBM.  L2 is flushed (a 256 MiB write) before each
timed step and each step is timed alone with CUDA events on the launching
stream.  Under torchrun every rank runs its own replica of the workload
(weak scaling, no data-path collective); the step time is the max over ranks.

``--profile-once`` makes one call of each stage entry point (dsa_index_scores,
dsa_topk_set, dsa_sparse_attend) on the workload and exits, timing nothing: the
command an ncu capture of the three stage kernels runs.

``--impl reference`` times the CPU oracle (the reference arm for this build)
on a bounded sample of the same workload and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "DSA layer query-tokens/sec (prefill & decode, top_k=2048); % of roofline"
UNIT = "query-tokens/s"
L2_FLUSH_BYTES = 256 << 20


# --------------------------------------------------------------------- peaks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ------------------------------------------------------------ algorithmic work
def visible_counts(wl):
    qp = wl["q_pos"].long()
    ks = wl["kv_start"].long().view(-1, 1)
    kl = wl["kv_len"].long().view(-1, 1)
    hi = torch.minimum(qp, kl - 1)
    return (hi - ks + 1).clamp(min=0)


def work(wl):
    """Algorithmic FLOPs / bytes of each stage for one step of a token-mode workload."""
    nvis = visible_counts(wl)
    pairs_idx = int(nvis.sum())
    pairs_att = int(nvis.clamp(max=wl.top_k).sum())
    esz = 2 if wl.dtype == "bf16" else 4
    rows = wl.batch * wl.n_q
    return {
        "index_flop": 2.0 * pairs_idx * wl.idx_heads * wl.idx_dim,
        # k_I read once per sequence, q_I and w read, visible fp32 scores written
        "index_bytes": wl.batch * wl.n_kv * wl.idx_dim * esz + rows * wl.idx_heads * (wl.idx_dim * esz + 4)
        + 4.0 * pairs_idx,
        "topk_bytes": 4.0 * pairs_idx + 4.0 * rows * wl.top_k,
        "attend_flop": 2.0 * pairs_att * wl.heads * (wl.kd + wl.vd),
        # one gathered latent row per (query, selected key), q read, out written
        "attend_bytes": float(pairs_att) * wl.kd * esz + rows * wl.heads * (wl.kd + wl.vd) * esz,
        "rows": rows,
    }


# -------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, sampled every 5 ms in a thread
    through NVML (the device is found by its PCI bus id, so CUDA_VISIBLE_DEVICES cannot confuse
    it), else through nvidia-smi every 200 ms.  Reading only: no setting is touched."""

    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20), ("hw_thermal_slowdown", 0x40),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        pr = torch.cuda.get_device_properties(device_index)
        self.bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
        self.samples = []            # (sm_mhz, max_mhz, reason names)
        self.stop = threading.Event()
        self.proc = None
        self.source = None

    def __enter__(self):
        try:
            import pynvml as N
            N.nvmlInit()
            h = N.nvmlDeviceGetHandleByPciBusId(self.bus.encode())
            mx = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)

            def run():
                while not self.stop.is_set():
                    try:
                        sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
                        r = N.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((float(sm), float(mx), [n for n, b in self.REASONS if r & b]))
                    except Exception:
                        pass
                    self.stop.wait(0.005)
            self.source = "nvml"
            self.t = threading.Thread(target=run, daemon=True)
            self.t.start()
            return self
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.bus}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
            self.t = threading.Thread(target=self._read_smi, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read_smi(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 9:
                continue
            try:
                self.samples.append((float(parts[1]), float(parts[2]),
                                     [n for n, v in zip(names, parts[5:9]) if v.lower() == "active"]))
            except ValueError:
                continue

    def __exit__(self, *a):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        elif self.source == "nvml":
            self.t.join(timeout=1)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        reasons = sorted({n for _, _, rs in self.samples for n in rs})
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples), "reasons": reasons,
                "samples": len(self.samples), "source": self.source, "gpu": self.bus}


# --------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
        return dist.get_rank(), world, int(os.environ.get("LOCAL_RANK", "0"))
    return 0, 1, 0


def replica_seed(workload: str, rank: int):
    """Seed of this rank's replica: rank 0 runs the standard workload, others their own draw."""
    return None if rank == 0 else 1000 + rank


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------ the CUDA path
def device_inputs(wl):
    return {k: v.cuda(non_blocking=False) for k, v in wl.tensors.items()}


def layer_args(wl, t):
    from sparse_attention_sum_b200 import runner
    lat = t["latent"]
    dims = runner.layer_dims(t["q_idx"], t["k_idx"], t["q"], lat, wl.vd, wl.top_k)
    args = dict(q_idx=t["q_idx"], k_idx=t["k_idx"], w=t["w"], idx_scale=wl.idx_scale, q_pos=t["q_pos"],
                kv_start=t["kv_start"], kv_len=t["kv_len"], q=t["q"], k=lat, v=lat,
                attn_scale=wl.attn_scale, k_row_stride=wl.kd, v_row_stride=wl.kd)
    return dims, args


def time_steps(step_fn, steps, warmup, flush, stream):
    """Each step timed alone on `stream` with CUDA events; L2 flushed in between."""
    for _ in range(warmup):
        step_fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush.fill_(1)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step_fn()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1) / 1e3)
    return times


def stage_times(wl, t, dims, args, bufs, steps, flush, stream):
    """Per-stage device times (s) of the three C-ABI calls the fused layer makes."""
    import sparse_attention_sum_b200 as dsa
    B, T, S = wl.batch, wl.n_q, wl.n_kv
    scores = bufs.ws[: B * T * S * 4].view(torch.float32)
    idx = bufs.idx
    calls = {
        "index": lambda: dsa.index_scores(dims, args["q_idx"], args["k_idx"], args["w"], args["idx_scale"],
                                          args["q_pos"], args["kv_start"], args["kv_len"], scores),
        # the fused layer's form of the selection (the set in key order, no rank sort)
        "topk": lambda: dsa.topk_set(dims, scores, args["q_pos"], args["kv_start"], args["kv_len"], wl.top_k,
                                     idx),
        "attend": lambda: dsa.sparse_attend(dims, args["q"], args["k"], args["k_row_stride"], args["v"],
                                            args["v_row_stride"], idx, wl.top_k, args["attn_scale"],
                                            bufs.out),
    }
    res = {}
    for name, fn in calls.items():
        ts = time_steps(fn, max(3, steps), 2, flush, stream)
        res[name] = statistics.median(ts)
    return res


def roofline_entry(kind, amount, seconds, peaks, traffic=None):
    if kind == "tensor":
        achieved = amount / seconds / 1e12
        peak = peaks["bf16_tflops"]
        sustained = peaks["bf16_tflops_sustained"]
        return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_source": peaks["source"] + " (burst)",
                "peak_sustained": sustained, "frac_sustained": round(achieved / sustained, 4)}
    achieved = amount / seconds / 1e9
    peak = peaks["hbm_gbs"]
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": peaks["source"]}


def profiled_traffic():
    """Per-launch DRAM traffic from the committed ncu summaries (profiles/traffic.txt), keyed by
    kernel:workload; an entry whose kernel source changed since the capture is dropped."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    res = {}
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return res
    for ln in lines:
        parts = ln.split()
        if not parts or parts[0].startswith("#") or len(parts) < 4:
            continue
        key, nbytes, src, digest = parts[:4]
        try:
            cur = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()[:16]
        except OSError:
            continue
        if cur == digest:
            res[key] = int(nbytes)
    return res


def profile_once(a):
    """One call of each entry point of the chosen path, no timing (for a profiler to capture).
    --what layer: dsa_index_scores, dsa_topk_set, dsa_sparse_attend; fused: dsa_index_topk; fp8:
    dsa_fp8_quantize of the queries, dsa_index_scores_fp8, dsa_index_topk_fp8 (keys quantised first);
    rotate: dsa_index_rotate of T tokens x 64 query heads, then of T keys."""
    import sparse_attention_sum_b200 as dsa
    from sparse_attention_sum_b200 import runner
    torch.cuda.set_device(0)
    dsa.lib()
    if a.what == "rotate":
        n = a.T or 4096
        qi = {k: v.cuda() for k, v in workloads.rotate_inputs(n, 64, 128, seed=1, pos_max=n).items()}
        ki = {k: v.cuda() for k, v in workloads.rotate_inputs(n, 1, 128, seed=2, pos_max=n, mean=0.5, std=2.0).items()}
        q_out = torch.empty(n, 64, 128, dtype=torch.bfloat16, device="cuda")
        k_out = torch.empty(n, 1, 128, dtype=torch.bfloat16, device="cuda")
        dsa.index_rotate(qi["x"], q_out, 64, 10000.0, pos=qi["pos"])
        dsa.index_rotate(ki["x"], k_out, 64, 10000.0, pos=ki["pos"], layer_norm=True, ln_w=ki["ln_w"], ln_b=ki["ln_b"],
                         ln_eps=1e-6)
        name = f"rotate T={n}"
    else:
        sizes = {k: v for k, v in (("T", a.T), ("S", a.S), ("B", a.B)) if v}
        wl = workloads.make(a.workload, **sizes)
        t = device_inputs(wl)
        dims, args = layer_args(wl, t)
        bufs = runner.LayerBuffers(dims, "cuda", torch.bfloat16, with_idx=True)
        B, T, S = wl.batch, wl.n_q, wl.n_kv
        scores = bufs.ws[: B * T * S * 4].view(torch.float32)
        ia = (args["q_pos"], args["kv_start"], args["kv_len"])
        if a.what == "layer":
            dsa.index_scores(dims, args["q_idx"], args["k_idx"], args["w"], args["idx_scale"], *ia, scores)
            dsa.topk_set(dims, scores, *ia, wl.top_k, bufs.idx)
            dsa.sparse_attend(dims, args["q"], args["k"], args["k_row_stride"], args["v"], args["v_row_stride"],
                              bufs.idx, wl.top_k, args["attn_scale"], bufs.out)
        elif a.what == "fused":
            dsa.index_topk(dims, args["q_idx"], args["k_idx"], args["w"], args["idx_scale"], *ia, wl.top_k, bufs.idx)
        elif a.what == "fp8":
            kc = torch.empty(B, S, 128, dtype=torch.uint8, device="cuda")
            ks = torch.empty(B, S, dtype=torch.float32, device="cuda")
            dsa.fp8_quantize(t["k_idx"], kc, ks)
            f8 = runner.Fp8Buffers(dims, "cuda")
            dsa.fp8_quantize(t["q_idx"], f8.q_codes, f8.q_scales)
            dsa.index_scores_fp8(dims, f8.q_codes, f8.q_scales, kc, ks, args["w"], args["idx_scale"], *ia, scores)
            dsa.index_topk_fp8(dims, f8.q_codes, f8.q_scales, kc, ks, args["w"], args["idx_scale"], *ia, wl.top_k,
                               bufs.idx)
        name = wl.name
    torch.cuda.synchronize()
    status = dsa.get_device_status()
    print(json.dumps({"profile_once": name, "what": a.what, "device_status": status,
                      "device_bytes": torch.cuda.max_memory_allocated()}), flush=True)
    if status != 0:
        sys.exit(1)


def run_ours(a):
    import sparse_attention_sum_b200 as dsa
    from sparse_attention_sum_b200 import runner

    rank, world, local = dist_setup(a.gpus)
    torch.cuda.set_device(local)
    dsa.lib()
    peaks = measured_peaks()
    wl = workloads.make(a.workload, seed=replica_seed(a.workload, rank))
    t = device_inputs(wl)
    dims, args = layer_args(wl, t)
    bufs = runner.LayerBuffers(dims, "cuda", torch.bfloat16, with_idx=True)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    step = lambda: runner.dsa_layer(dims, **args, bufs=bufs)

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        times = time_steps(step, a.steps, a.warmup, flush, stream)
    barrier(world)
    torch.cuda.synchronize()
    total = max_over_ranks(sum(times), world)
    assert dsa.get_device_status() == 0, "device reported a bounded-wait timeout"
    rows = wl.batch * wl.n_q
    value = world * rows * a.steps / total
    wk = work(wl)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(1e3 * total / a.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32",
        "data": "synthetic (seeded CPU generator, bf16)",
        "config": {"workload": f"{wl.name}: B={wl.batch} T={wl.n_q} S={wl.n_kv} top_k={wl.top_k} "
                               f"indexer {wl.idx_heads}x{wl.idx_dim}, MLA H={wl.heads} kd={wl.kd} vd={wl.vd}",
                   "l2": "flushed (256 MiB write) before every timed step",
                   "parallelism": f"replicas x{world} (one independent problem per GPU)"},
        "gpu_launches": 3 * a.steps,   # index, top-k set, attend per fused layer step
        "clocks": clk.summary(),
    }
    if not a.no_extras:
        # every rank: end to end through the public API on its own replica (collective: barrier, max)
        line["e2e"] = e2e_measure(wl, a.steps, stream, world)
    if rank == 0 and not a.no_extras:
        st = stage_times(wl, t, dims, args, bufs, 5, flush, stream)
        step_med = statistics.median(times)
        line["stages_us"] = {k: round(v * 1e6, 1) for k, v in st.items()}
        line["stages_qtok_s"] = {k: round(rows / v, 1) for k, v in st.items()}
        line["fused_tensor_frac"] = round((wk["index_flop"] + wk["attend_flop"]) / step_med / 1e12
                                          / peaks["bf16_tflops"], 4)
        tr = profiled_traffic()
        traffic = tr.get(f"attend:{wl.name}")
        line["roofline"] = roofline_entry("tensor", wk["attend_flop"], st["attend"], peaks, traffic)
        line["roofline"]["kernel"] = "sparse attend (dsa_sparse_attend)"
        line["fp8_indexer"] = fp8_indexer_extra(wl, t, dims, args, bufs, peaks, flush, stream, 5)
        line["roofline_stages"] = {
            "index": roofline_entry("tensor", wk["index_flop"], st["index"], peaks, tr.get(f"index:{wl.name}")),
            "topk": roofline_entry("hbm", wk["topk_bytes"], st["topk"], peaks, tr.get(f"topk:{wl.name}")),
            "attend": roofline_entry("tensor", wk["attend_flop"], st["attend"], peaks, traffic),
        }
    if rank == 0 and not a.no_extras and world == 1:
        # IndexShare: a layer that reuses an earlier layer's selection runs only the attend.  On the
        # 78-layer stack the pages describe, layers 0, 1 and every il % 4 == 2 compute their own (21 of 78).
        shared = time_steps(lambda: runner.dsa_layer(dims, **args, bufs=bufs, idx_in=bufs.idx), max(3, a.steps // 2),
                            3, flush, stream)
        full_ms, shared_ms = statistics.median(times) * 1e3, statistics.median(shared) * 1e3
        n_full = sum(1 for il in range(78) if runner.computes_own_selection(il))
        stack_ms = (n_full * full_ms + (78 - n_full) * shared_ms) / 78
        line["indexshare"] = {"shared_layer_ms": round(shared_ms, 4), "full_layer_ms": round(full_ms, 4),
                              "layers_full_of_78": n_full, "stack_avg_layer_ms": round(stack_ms, 4),
                              "stack_avg_value": round(rows / (stack_ms / 1e3), 1), "unit": UNIT}
        if a.workload == "prefill":
            line["decode"] = decode_extra(peaks, flush, stream, a.cpu_seconds / 2)
            line["chunked"] = chunked_extra(peaks, flush, stream, a.cpu_seconds / 3)
            line["kpool"] = kpool_extra(peaks, flush, stream, a.cpu_seconds / 3)
            line["rotate"] = rotate_extra(peaks, flush, stream)
        line["cpu_baseline"] = cpu_baseline(wl, budget_s=a.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del t, bufs
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def e2e_measure(wl, steps, stream, world=1):
    """Same metric through the public API with host buffers.  Every step copies its inputs from
    pinned host memory to the device, runs the fused layer and reads its output back to pinned
    host memory, all inside the timed region.  Steps are pipelined the way a serving loop runs
    them: step i+1's upload (one copy stream) overlaps step i's layer (the compute stream) and
    step i-1's download (a second copy stream); two device buffer sets alternate.  With several
    ranks each runs its own replica between barriers; the rate is the whole job's over the
    slowest rank."""
    from sparse_attention_sum_b200 import runner
    host = {k: v.pin_memory() for k, v in wl.tensors.items()}
    sets = []
    for _ in range(2):
        dev_t = {k: torch.empty_like(v, device="cuda") for k, v in host.items()}
        dims, args = layer_args(wl, dev_t)
        bufs = runner.LayerBuffers(dims, "cuda", torch.bfloat16, with_idx=True)
        sets.append((dev_t, dims, args, bufs))
    out_host = torch.empty(sets[0][3].out.shape, dtype=sets[0][3].out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host.numel() * out_host.element_size()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    downloaded = [torch.cuda.Event() for _ in range(2)]
    for e in downloaded:
        e.record(down)

    def run(n):
        for i in range(n):
            b = i & 1
            dev_t, dims, args, bufs = sets[b]
            with torch.cuda.stream(up):
                up.wait_event(computed[b]) if i >= 2 else None     # set b's inputs are free again
                for k in host:
                    dev_t[k].copy_(host[k], non_blocking=True)
                uploaded[b].record(up)
            stream.wait_event(uploaded[b])
            stream.wait_event(downloaded[b])                        # set b's output was read back
            runner.dsa_layer(dims, **args, bufs=bufs, stream=stream)
            computed[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                out_host.copy_(bufs.out, non_blocking=True)
                downloaded[b].record(down)

    run(2)
    torch.cuda.synchronize()
    barrier(world)
    n = max(4, min(steps, 10))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(up)
    run(n)
    down.wait_event(computed[(n - 1) & 1])
    e1.record(down)
    e1.synchronize()
    sec = max_over_ranks(e0.elapsed_time(e1) / 1e3 / n, world)
    return {"value": round(world * wl.batch * wl.n_q / sec, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(sec * 1e3, 3),
            "pipelined": "upload of step i+1 and download of step i-1 overlap step i's layer"}


def fp8_indexer_extra(wl, t, dims, args, bufs, peaks, flush, stream, steps):
    """The FP8 indexer on this workload: keys quantised once (a cache holds them as e4m3 codes), then per
    step the queries are quantised and scored (dsa_fp8_quantize + dsa_index_scores_fp8), and the layer
    chain runner.dsa_layer_fp8 (quantise, FP8 scores, top-k set, attend) is timed whole."""
    import sparse_attention_sum_b200 as dsa
    from sparse_attention_sum_b200 import runner
    B, T, S = wl.batch, wl.n_q, wl.n_kv
    k_codes = torch.empty(B, S, 128, dtype=torch.uint8, device="cuda")
    k_scales = torch.empty(B, S, dtype=torch.float32, device="cuda")
    dsa.fp8_quantize(t["k_idx"], k_codes, k_scales)
    fp8 = runner.Fp8Buffers(dims, "cuda")
    scores = bufs.ws[: B * T * S * 4].view(torch.float32)
    quant = lambda: dsa.fp8_quantize(t["q_idx"], fp8.q_codes, fp8.q_scales)
    index = lambda: dsa.index_scores_fp8(dims, fp8.q_codes, fp8.q_scales, k_codes, k_scales, args["w"],
                                         args["idx_scale"], args["q_pos"], args["kv_start"], args["kv_len"], scores)
    t_quant = statistics.median(time_steps(quant, max(3, steps), 2, flush, stream))
    t_index = statistics.median(time_steps(index, max(3, steps), 2, flush, stream))
    layer = statistics.median(time_steps(
        lambda: runner.dsa_layer_fp8(dims, k_codes=k_codes, k_scales=k_scales, bufs=bufs, fp8=fp8, **args),
        max(3, steps), 3, flush, stream))
    nvis = visible_counts(wl)
    pairs = int(nvis.sum())
    rows = B * T
    fp8_peaks = dict(peaks, bf16_tflops=2 * peaks["bf16_tflops"],
                     bf16_tflops_sustained=2 * peaks["bf16_tflops_sustained"],
                     source=peaks["source"] + " bf16 x 2 (dense e4m3 : bf16 nominal ratio)")
    idx_bytes = B * S * (128 + 4) + rows * wl.idx_heads * (128 + 4 + 4) + 4.0 * pairs
    res = {"layer_ms": round(layer * 1e3, 4), "value": round(rows / layer, 1), "unit": UNIT,
           "stages_us": {"quantize_q": round(t_quant * 1e6, 2), "index_fp8": round(t_index * 1e6, 1)},
           "roofline_index_fp8": roofline_entry("tensor", 2.0 * pairs * wl.idx_heads * wl.idx_dim, t_index,
                                                fp8_peaks),
           "roofline_index_fp8_hbm": roofline_entry("hbm", idx_bytes, t_index, peaks),
           "roofline_quantize_q": roofline_entry("hbm", rows * wl.idx_heads * (256 + 128 + 4), t_quant, peaks)}
    del k_codes, k_scales, fp8
    return res


def fused_select_extra(wl, t, dims, args, bufs, peaks, flush, stream, steps):
    """The selection without a score matrix (dsa_index_topk, and dsa_index_topk_fp8 on a key cache held as
    e4m3 codes), alone and followed by the sparse attend, against the two-kernel selection."""
    import sparse_attention_sum_b200 as dsa
    from sparse_attention_sum_b200 import runner
    B, T, S = wl.batch, wl.n_q, wl.n_kv
    rows = B * T
    a = args
    k_codes = torch.empty(B, S, 128, dtype=torch.uint8, device="cuda")
    k_scales = torch.empty(B, S, dtype=torch.float32, device="cuda")
    dsa.fp8_quantize(t["k_idx"], k_codes, k_scales)
    fp8 = runner.Fp8Buffers(dims, "cuda")
    sel = lambda: dsa.index_topk(dims, a["q_idx"], a["k_idx"], a["w"], a["idx_scale"], a["q_pos"], a["kv_start"],
                                 a["kv_len"], wl.top_k, bufs.idx)

    def sel8():
        dsa.fp8_quantize(t["q_idx"], fp8.q_codes, fp8.q_scales)
        dsa.index_topk_fp8(dims, fp8.q_codes, fp8.q_scales, k_codes, k_scales, a["w"], a["idx_scale"], a["q_pos"],
                           a["kv_start"], a["kv_len"], wl.top_k, bufs.idx)
    att = lambda: dsa.sparse_attend(dims, a["q"], a["k"], a["k_row_stride"], a["v"], a["v_row_stride"], bufs.idx,
                                    wl.top_k, a["attn_scale"], bufs.out)
    med = lambda f: statistics.median(time_steps(f, max(3, steps), 3, flush, stream))
    t_sel, t_sel8 = med(sel), med(sel8)
    t_layer = med(lambda: (sel(), att()))
    t_layer8 = med(lambda: (sel8(), att()))
    nvis = int(visible_counts(wl).sum())
    sel_bytes = B * S * 256 + rows * wl.idx_heads * (256 + 4) + 4.0 * rows * wl.top_k
    sel8_bytes = B * S * (128 + 4) + rows * wl.idx_heads * (256 + 128 + 4 + 4 + 4) + 4.0 * rows * wl.top_k
    res = {"select_us": round(t_sel * 1e6, 1), "select_fp8_us": round(t_sel8 * 1e6, 1),
           "layer_ms": round(t_layer * 1e3, 4), "layer_value": round(rows / t_layer, 1),
           "layer_fp8_ms": round(t_layer8 * 1e3, 4), "layer_fp8_value": round(rows / t_layer8, 1), "unit": UNIT,
           "roofline_select": roofline_entry("hbm", sel_bytes, t_sel, peaks),
           "roofline_select_fp8": roofline_entry("hbm", sel8_bytes, t_sel8, peaks),
           "index_flop": 2.0 * nvis * wl.idx_heads * wl.idx_dim}
    del k_codes, k_scales, fp8
    return res


def decode_extra(peaks, flush, stream, cpu_s=0.0):
    """The decode workload (64 sequences x 1 query vs 32768 cached keys) and its stages."""
    from sparse_attention_sum_b200 import runner
    wl = workloads.make("decode")
    t = device_inputs(wl)
    dims, args = layer_args(wl, t)
    bufs = runner.LayerBuffers(dims, "cuda", torch.bfloat16, with_idx=True)
    times = time_steps(lambda: runner.dsa_layer(dims, **args, bufs=bufs), 10, 3, flush, stream)
    st = stage_times(wl, t, dims, args, bufs, 10, flush, stream)
    wk = work(wl)
    rows = wl.batch * wl.n_q
    step = statistics.median(times)
    res = {"workload": f"decode: B={wl.batch} T=1 S={wl.n_kv} top_k={wl.top_k}",
           "value": round(rows / step, 1), "unit": UNIT, "ms_per_step": round(step * 1e3, 4),
           "stages_us": {k: round(v * 1e6, 1) for k, v in st.items()},
           "roofline_attend": roofline_entry("hbm", wk["attend_bytes"], st["attend"], peaks,
                                             profiled_traffic().get("attend:decode")),
           "roofline_index": roofline_entry("hbm", wk["index_bytes"], st["index"], peaks,
                                            profiled_traffic().get("index:decode")),
           "fused_hbm_frac": round((wk["index_bytes"] + wk["topk_bytes"] + wk["attend_bytes"]) / step / 1e9
                                   / peaks["hbm_gbs"], 4)}
    res["fp8_indexer"] = fp8_indexer_extra(wl, t, dims, args, bufs, peaks, flush, stream, 10)
    res["fused_select"] = fused_select_extra(wl, t, dims, args, bufs, peaks, flush, stream, 10)
    if cpu_s > 0:
        res["cpu_baseline"] = cpu_baseline(wl, budget_s=cpu_s, whole=True)
    del t, bufs
    torch.cuda.empty_cache()
    return res


def chunked_extra(peaks, flush, stream, cpu_s=0.0):
    """Chunked prefill: 4096 queries at positions 28672..32767 against 32768 keys (hot-spot keys)."""
    from sparse_attention_sum_b200 import runner
    wl = workloads.make("chunked")
    t = device_inputs(wl)
    dims, args = layer_args(wl, t)
    bufs = runner.LayerBuffers(dims, "cuda", torch.bfloat16, with_idx=True)
    times = time_steps(lambda: runner.dsa_layer(dims, **args, bufs=bufs), 5, 3, flush, stream)
    st = stage_times(wl, t, dims, args, bufs, 5, flush, stream)
    wk = work(wl)
    rows = wl.batch * wl.n_q
    step = statistics.median(times)
    res = {"workload": f"chunked: B={wl.batch} T={wl.n_q} S={wl.n_kv} top_k={wl.top_k}",
           "value": round(rows / step, 1), "unit": UNIT, "ms_per_step": round(step * 1e3, 4),
           "stages_us": {k: round(v * 1e6, 1) for k, v in st.items()},
           "roofline_index": roofline_entry("tensor", wk["index_flop"], st["index"], peaks),
           "roofline_attend": roofline_entry("tensor", wk["attend_flop"], st["attend"], peaks),
           "fused_tensor_frac": round((wk["index_flop"] + wk["attend_flop"]) / step / 1e12 / peaks["bf16_tflops"], 4)}
    if cpu_s > 0:
        res["cpu_baseline"] = cpu_baseline(wl, budget_s=cpu_s)
    del t, bufs
    torch.cuda.empty_cache()
    return res


def kpool_extra(peaks, flush, stream, cpu_s=0.0):
    """The kpool NoPE layer (4 sequences x 8192 tokens, left padding, kpool 4, select_k 512, H=64
    absorbed into a 512-wide latent): every call of the chain timed alone, and the whole chain."""
    import sparse_attention_sum_b200 as dsa
    from sparse_attention_sum_b200 import runner
    wl = workloads.make("kpool")
    t = device_inputs(wl)
    B, T, S = wl.batch, wl.n_q, wl.n_kv
    H, L = wl.heads, wl.kd
    dq, dv = t["q_nope"].shape[-1], t["w_uv"].shape[1]
    dims = runner.kpool_dims(B, T, S, wl.idx_heads, wl.idx_dim, wl.kpool, wl.select_k, wl.out_width, H, L)
    bufs = runner.KpoolBuffers(B, T, S, wl.idx_heads, wl.idx_dim, wl.kpool, wl.select_k, wl.out_width,
                               H, dq, L, dv, "cuda")
    dp, di, da = dims["pool"], dims["index"], dims["attend"]
    chain = lambda: runner.kpool_layer(dims, t["q_idx"], t["k_raw"], t["gate"], t["ln_w"], t["ln_b"], wl.ln_eps,
                                       t["w"], wl.idx_scale, t["q_pos"], t["kv_start"], t["kv_len"], t["q_nope"],
                                       t["latent"], t["w_uk"], t["w_uv"], wl.attn_scale, bufs)
    times = time_steps(chain, 3, 3, flush, stream)
    calls = {
        "pool_states": lambda: dsa.pool_states(dp, t["k_raw"], t["gate"], t["ln_w"], t["ln_b"], wl.ln_eps,
                                               t["kv_start"], t["kv_len"], bufs.pooled, bufs.n_pools),
        "index": lambda: dsa.index_scores(di, t["q_idx"], bufs.pooled, t["w"], wl.idx_scale, t["q_pos"],
                                          t["kv_start"], t["kv_len"], bufs.pool_scores),
        "topk": lambda: dsa.topk_set(di, bufs.pool_scores, t["q_pos"], t["kv_start"], t["kv_len"], di.top_k,
                                     bufs.pool_idx),
        "expand": lambda: dsa.expand_selection(dp, bufs.pool_idx, t["q_pos"], t["kv_start"], t["kv_len"],
                                               bufs.n_pools, bufs.tok_idx),
        "absorb_q": lambda: dsa.absorb_q(da, t["q_nope"], dq, t["w_uk"], L, bufs.q_lat),
        "attend": lambda: dsa.sparse_attend(da, bufs.q_lat, t["latent"], L, t["latent"], L, bufs.tok_idx,
                                            da.out_width, wl.attn_scale, bufs.o_lat),
        "absorb_out": lambda: dsa.absorb_out(da, bufs.o_lat, L, t["w_uv"], dv, bufs.out),
    }
    st = {k: statistics.median(time_steps(f, 3, 1, flush, stream)) for k, f in calls.items()}
    # the ranked selection of the same pools (dsa_topk), which the layer does not need
    ranked = torch.empty_like(bufs.pool_idx)
    topk_ranked = statistics.median(time_steps(
        lambda: dsa.topk(di, bufs.pool_scores, t["q_pos"], t["kv_start"], t["kv_len"], di.top_k, ranked),
        3, 1, flush, stream))
    del ranked
    index_pairs = int(torch.isfinite(bufs.pool_scores).sum())
    attend_pairs = int((bufs.tok_idx >= 0).sum())
    valid_rows = int((t["q_pos"] >= t["kv_start"].view(-1, 1)).sum())
    flop = {"index": 2.0 * index_pairs * wl.idx_heads * wl.idx_dim,
            "attend": 2.0 * attend_pairs * H * (L + L),
            "absorb": 2 * (2.0 * B * T * H * dq * L)}
    step = statistics.median(times)
    res = {"workload": f"kpool: B={B} T=S={S} left pad {wl['kv_start'].tolist()} kpool={wl.kpool} "
                       f"select_k={wl.select_k} width={wl.out_width}, NoPE MLA H={H} latent {L}",
           "value": round(B * T / step, 1), "value_valid_rows": round(valid_rows / step, 1), "unit": UNIT,
           "ms_per_step": round(step * 1e3, 3), "stages_us": {k: round(v * 1e6, 1) for k, v in st.items()},
           "topk_ranked_us": round(topk_ranked * 1e6, 1),
           "roofline_index": roofline_entry("tensor", flop["index"], st["index"], peaks),
           "roofline_attend": roofline_entry("tensor", flop["attend"], st["attend"], peaks),
           "roofline_absorb": roofline_entry("tensor", flop["absorb"], st["absorb_q"] + st["absorb_out"], peaks),
           "fused_tensor_frac": round(sum(flop.values()) / step / 1e12 / peaks["bf16_tflops"], 4)}
    if cpu_s > 0:
        res["cpu_baseline"] = cpu_baseline(wl, budget_s=cpu_s, row_fn=oracle_kpool_rows)
    del t, bufs
    torch.cuda.empty_cache()
    return res


def rotate_extra(peaks, flush, stream):
    """Indexer query / key preparation (dsa_index_rotate) for the prefill and decode layers.  Prefill
    rotates 4096 tokens x 64 query heads and writes 4096 LayerNorm-ed keys; decode rotates 64 x 64 query
    heads and appends one key per sequence at position 32767 of a 64 x 32768 key cache.  RoPE base 10000
    (the cost does not depend on it)."""
    import sparse_attention_sum_b200 as dsa
    theta, res = 10000.0, {}
    for name, n, S in (("prefill", 4096, 0), ("decode", 64, 32768)):
        qi = {k: v.cuda() for k, v in workloads.rotate_inputs(n, 64, 128, seed=1, pos_max=S or n).items()}
        ki = {k: v.cuda() for k, v in workloads.rotate_inputs(n, 1, 128, seed=2, pos_max=S or n, mean=0.5,
                                                                std=2.0).items()}
        q_out = torch.empty(n, 64, 128, dtype=torch.bfloat16, device="cuda")
        if S:
            cache = torch.zeros(n * S, 1, 128, dtype=torch.bfloat16, device="cuda")
            slots = torch.arange(n, dtype=torch.int32, device="cuda") * S + (S - 1)
            ki["pos"].fill_(S - 1)
        else:
            cache, slots = torch.empty(n, 1, 128, dtype=torch.bfloat16, device="cuda"), None
        qf = lambda: dsa.index_rotate(qi["x"], q_out, 64, theta, pos=qi["pos"])
        kf = lambda: dsa.index_rotate(ki["x"], cache, 64, theta, pos=ki["pos"], layer_norm=True, ln_w=ki["ln_w"],
                                      ln_b=ki["ln_b"], ln_eps=1e-6, out_rows=slots)
        tq = statistics.median(time_steps(qf, 10, 3, flush, stream))
        tk = statistics.median(time_steps(kf, 10, 3, flush, stream))
        q_bytes = 2 * n * 64 * 128 * 2 + 4 * n           # read and write every query value, positions
        k_bytes = 2 * n * 128 * 2 + 4 * n * (2 if S else 1) + 2 * 128 * 4
        res[name] = {"rows": n, "queries_us": round(tq * 1e6, 2), "keys_us": round(tk * 1e6, 2),
                     "roofline_queries": roofline_entry("hbm", q_bytes, tq, peaks),
                     "roofline_keys": roofline_entry("hbm", k_bytes, tk, peaks)}
        del qi, ki, q_out, cache
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------ the CPU oracle
def oracle_rows(wl, rows):
    from oracle import dsa_oracle as O
    lat = wl["latent"]
    K, V = lat.unsqueeze(2), lat[..., :wl.vd].unsqueeze(2)
    ts = wl.tensors
    for b, t in rows:
        O.layer_row(b, t, ts, wl.top_k, wl.idx_scale, wl.attn_scale, wl["q"], K, V)


def oracle_kpool_rows(wl, rows, _pooled={}):
    """The kpool layer row by row in the oracle: pooled keys of the row's sequence (once per
    sequence), pool scores and top-k, expand_selection, then the literal expand_kv attention."""
    from oracle import dsa_oracle as O
    for b, t in rows:
        f, L = int(wl["kv_start"][b]), int(wl["kv_len"][b])
        key = (id(wl), b)
        if key not in _pooled:
            _pooled[key] = O.pool_states(wl["k_raw"][b], wl["gate"][b], f, L, wl.kpool, wl["ln_w"], wl["ln_b"],
                                         wl.ln_eps)
        pooled = _pooled[key]
        p = int(wl["q_pos"][b, t])
        sel, _ = O.topk_pools_row(wl["q_idx"][b, t], pooled, wl["w"][b, t], wl.idx_scale, p, f, pooled.shape[0],
                                  wl.kpool, wl.select_k)
        tok = O.expand_selection(sel, p, f, L, wl.kpool, pooled.shape[0], wl.out_width)
        O.mla_masked_attention_row(wl["q_nope"][b, t], wl["latent"][b], wl["w_uk"], wl["w_uv"], tok,
                                   wl.attn_scale)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline(wl, budget_s=15.0, whole=False, row_fn=None):
    """Oracle query rows per second on this host: every row of the workload when ``whole`` (decode),
    else a bounded stratified sample (first, last and top-k boundary row of every sequence, then random
    rows until the time budget is spent)."""
    import random
    row_fn = row_fn or oracle_rows
    T = wl.n_q
    rnd = random.Random(0)
    t0 = time.perf_counter()
    if whole:
        rows = [(b, t) for b in range(wl.batch) for t in range(T)]
        row_fn(wl, rows)
        el = time.perf_counter() - t0
        return {"value": round(len(rows) / el, 3), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                "sample": f"all {len(rows)} query rows of {wl.name}, {el:.1f} s, f64 numpy oracle"}
    order = [(b, t) for b in range(wl.batch) for t in (0, T - 1, min(T - 1, wl.top_k))]
    done = 0
    while time.perf_counter() - t0 < budget_s and done < 4096:
        batch = order if done == 0 else [(rnd.randrange(wl.batch), rnd.randrange(T)) for _ in range(4)]
        row_fn(wl, batch)
        done += len(batch)
    el = time.perf_counter() - t0
    return {"value": round(done / el, 3), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{done} query rows of {wl.name} (first, last, top-k boundary, then random), "
                      f"{el:.1f} s, f64 numpy oracle, extrapolated per query row"}


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = workloads.make(a.workload)
    rows_per_step = 4
    import random
    rnd = random.Random(1)
    for _ in range(a.warmup):
        oracle_rows(wl, [(0, rnd.randrange(wl.n_q))])
    times = []
    for _ in range(a.steps):
        rows = [(rnd.randrange(wl.batch), rnd.randrange(wl.n_q)) for _ in range(rows_per_step)]
        t0 = time.perf_counter()
        oracle_rows(wl, rows)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = rows_per_step * a.steps / total
    cores = blas_threads()
    line = {"metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": 1, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": round(1e3 * total / a.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded CPU generator, bf16)",
            "config": {"workload": f"{wl.name}: B={wl.batch} T={wl.n_q} S={wl.n_kv} top_k={wl.top_k}",
                       "sample": f"{rows_per_step} random query rows per step"},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{rows_per_step} random query rows of {wl.name} per step"},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill", "decode", "chunked"], default="prefill")
    ap.add_argument("--no-extras", action="store_true", help="skip stages, decode, e2e and CPU baseline")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--profile-once", action="store_true",
                    help="one call of each stage entry point, no timing (for an ncu capture)")
    ap.add_argument("--T", type=int, default=0, help="--profile-once: queries per sequence (smaller capture)")
    ap.add_argument("--S", type=int, default=0, help="--profile-once: keys per sequence (smaller capture)")
    ap.add_argument("--B", type=int, default=0, help="--profile-once: sequences (decode; smaller capture)")
    ap.add_argument("--what", choices=["layer", "fused", "fp8", "rotate"], default="layer",
                    help="--profile-once: which path to run once")
    a = ap.parse_args(argv)
    a.warmup = max(3, a.warmup)  # at least three untimed warm-up steps
    if a.impl == "reference":
        run_reference(a)
    elif a.profile_once:
        profile_once(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
