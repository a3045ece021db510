"""Benchmark: MoE-layer tokens/s of the W4A16 quantised MoE layer on B200.

One step = one pass of the whole hot path over one batch: moe_route_permute
(router, optional bit gate, histogram, scan, permutation, gather) ->
moe_grouped_ffn_combine (dequant-fused gate/up + SwiGLU, then down, then the
weighted combine).  The FFN-only timing behind the roofline figure runs
moe_grouped_ffn_wq alone.
Default workload: the OLMoE-shaped layer (d=2048, E=64, top-8, d_ff=1024,
INT4 g128, Zipf-skewed router bias) at T=4096 tokens.  Synthetic seeded
inputs and random weights; R distinct layer instances are rotated so the
expert weights streamed per step are not L2-resident.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank runs an
independent replica on its own token batch (the layer has no exchange step
in this data-parallel form); time = max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import threading
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (W4A16)"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="olmoe")
    p.add_argument("--tokens", type=int, default=4096)
    p.add_argument("--instances", type=int, default=4, help="distinct layer instances rotated per step")
    p.add_argument("--sweep", default="1,8,16,256", help="extra token counts timed for context ('' = none)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sample-tokens", type=int, default=0)
    p.add_argument("--workloads", default="mixtral:8192,mixtral:512,mixtral:32,mixtral:1,nested:2048,nested:64,"
                                          "nested:1,nested_gate:2048,nested_gate:1,tiny:64",
                   help="other configured workloads reported for context (name:tokens,...; '' = none)")
    p.add_argument("--offload-steps", type=int, default=512,
                   help="decode steps of the offload (slot-cache) workload reported under 'offload', after "
                        "16 warm-up steps, per schedule (0 = skip)")
    p.add_argument("--profile", action="store_true",
                   help="profiling driver: one instance, warmup + steps of the eager step, no JSON")
    return p.parse_args()


# ------------------------------------------------------------------ util --

def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value):
    """The largest of the ranks' values (every rank gets it)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_step, steps, max_ms):
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    return world * units_per_step * steps / (max_ms / 1e3)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], tc=p["bf16_tflops"], tc_sust=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    src="measured")
    return dict(hbm=6650.0, tc=1590.0, tc_sust=1400.0, src="fallback")


class ClockSampler:
    """SM clock and throttle reasons sampled every few milliseconds (NVML, in
    a thread) while the timed region runs; nvidia-smi polling if NVML is not
    importable."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.thread = None
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.stop_flag = False

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            pr = torch.cuda.get_device_properties(self.gpu)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons

            def run():
                while not self.stop_flag:
                    try:
                        self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                        r = int(get_reasons(h))
                        for n, bit in self.REASONS.items():
                            if r & bit:
                                self.reasons.add(n)
                    except Exception:
                        pass
                    time.sleep(0.005)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=2)
            if not self.samples:
                return None
            return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                    "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi"}


# -------------------------------------------------------------- workload --

def make_instances(shape, T, R, seed, device, bit_gate=False):
    """R layer instances with weights drawn and packed on the device.  With
    bit_gate (nested-plane layout), each instance gets a bit-width gate and
    its widths are chosen on the device every step (moe_bit_gate) instead of
    being drawn from the seed."""
    import torch
    from quantized_moe_expert_histogram_b200 import inputs as I
    from quantized_moe_expert_histogram_b200.layer import QuantMoELayer
    layers = []
    for r in range(R):
        L = I.make_layer(shape, T, seed=seed + 1000 * r, device=device)
        layer = QuantMoELayer.from_weights(shape, L["w_router"], L["bias"], L["w_gate"], L["w_up"],
                                           L["w_down"], max_tokens=T)
        del L["w_gate"], L["w_up"], L["w_down"]
        torch.cuda.empty_cache()
        bits = L.get("bits")
        if bit_gate:
            G = I.make_bit_gate(shape, seed=seed + 1000 * r + 1, device=device, bias=True)
            layer.w_bit, layer.bias_bit = G["w_bit"], G["bias_bit"]
            bits = None
        layers.append((layer, L["x"], bits))
    return layers


def kernel_launches(shape, T, bit_gate=False):
    """Kernels of this library launched by one layer step, following the
    library's own choices: router, bit gate and permutation as one cluster
    launch for the smallest batches (T <= 8, T*E <= 512, with a bit gate
    T*E <= 128, T*k <= 64, d % 256 == 0); otherwise router 1 (one cluster
    launch under the same rule on T*E) or 2, bit gate 1 when used, permutation 1 (single CTA,
    with the gather when it is small) or 1 + gather, or 3 + gather; then
    FFN 2 and the combine 1."""
    n = T * shape.k
    comb = 1
    if T <= 8 and T * shape.E <= (128 if bit_gate else 512) and n <= 64 and shape.d % 256 == 0:
        return 1 + 2 + comb
    nbins = shape.E * (3 if shape.layout == "planes" else 1)
    route = 1 if (T <= 8 and T * shape.E <= 512 and shape.d % 256 == 0) else 2
    if n <= 1024:
        perm = 1 if n * shape.d <= 64 * 1024 else 2
    else:
        perm = 4
    del nbins
    return route + (1 if bit_gate else 0) + perm + 2 + comb


def profiled_traffic(workload, T):
    """DRAM bytes (read + write) of one FFN call (gate/up + down launches) from
    the committed ncu summary, if it covers this workload and the kernel
    source is unchanged since the counters were taken; else None."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", f"k_ffn_tc_{workload}_t{T}.md")
    src = os.path.join(ROOT, "quantized_moe_expert_histogram_b200", "csrc", "tc_gemm.cu")
    if not os.path.exists(path):
        return None, None
    text = open(path).read()
    m_hash = re.search(r"source_sha1: ([0-9a-f]{40})", text)
    m_bytes = re.search(r"dram_bytes_per_step: (\d+)", text)
    if not m_hash or not m_bytes:
        return None, None
    with open(src, "rb") as f:
        if hashlib.sha1(f.read()).hexdigest() != m_hash.group(1):
            return None, "kernel changed since the ncu capture"
    return int(m_bytes.group(1)), os.path.relpath(path, ROOT)


def algorithmic(shape, T, layer, bits_present):
    """Algorithmic bytes and flops of one layer pass from the routing taken."""
    from quantized_moe_expert_histogram_b200 import moeq
    counts = layer.views(T)["counts"].cpu().tolist()
    d, F, g = shape.d, shape.F, shape.group
    code_full = 3 * d * F // 2
    sz = 3 * d * F // g * 4
    bytes_w = 0
    if not bits_present:
        bytes_w = sum(1 for c in counts if c > 0) * (code_full + sz)
    else:
        for e in range(shape.E):
            bs = [2 + j for j in range(3) if counts[3 * e + j] > 0]
            if bs:
                bytes_w += code_full * max(bs) // 4 + sz
    act = 2 * T * d * 2  # x in, y out (bf16)
    flops = 6 * d * F * T * shape.k
    return bytes_w + act, flops


def _step_calls(layer, x, bits, stream, part):
    """The ABI calls of one step: part 'all', or 'ffn' (the FFN call only)."""
    from quantized_moe_expert_histogram_b200 import moeq
    T = x.shape[0]
    v = layer.views(T)
    if part == "all":
        gate = bits is None and layer.w_bit is not None
        moeq.moe_route_permute(x, layer.w_router, layer.bias, layer.k, bits=bits,
                               w_bit=layer.w_bit if gate else None, bias_bit=layer.bias_bit if gate else None,
                               out=v, status=v["status"], workspace=v["rp_ws"], stream=stream)
    if part == "all":
        moeq.moe_grouped_ffn_combine(v["x_perm"], v["offsets"], layer.blobs, T, layer.k, layer.E, layer.d,
                                     layer.F, layer.group, layer.layout, v["perm"], v["inv_perm"], v["topk_w"],
                                     y=v["y"], y_perm=v["y_perm"], workspace=v["workspace"], status=v["status"],
                                     stream=stream)
    else:
        moeq.moe_grouped_ffn_wq(v["x_perm"], v["offsets"], layer.blobs, T, layer.E, layer.d, layer.F,
                                layer.group, layer.layout, workspace=v["workspace"], y_perm=v["y_perm"],
                                status=v["status"], stream=stream)


def capture(layers, stream, part):
    """One CUDA graph running the steps of all R instances back to back."""
    import torch
    for layer, x, bits in layers:  # eager pass first (sets kernel attributes, routing for 'ffn')
        _step_calls(layer, x, bits, stream, "all")
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for layer, x, bits in layers:
            _step_calls(layer, x, bits, stream, part)
    torch.cuda.synchronize()
    return g


def time_graph(g, replays, warmup, stream):
    import torch
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(replays):
            g.replay()
        end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def time_e2e(layers, steps, stream):
    """Same steps through the public layer call with pinned host buffers:
    every step's H2D of x and D2H of y inside the timed region, pipelined
    as a serving loop would run them: step i's input copy (copy stream 1)
    and step i-1's output copy (copy stream 2) overlap step i-1's / i's
    layer call (the compute stream), with events ordering each buffer's
    reuse (two device x buffers, two pinned y buffers; a layer instance's y
    is read out before that instance runs again)."""
    import torch
    R = len(layers)
    T, d = layers[0][1].shape
    hx = [layers[r][1].cpu().pin_memory() for r in range(R)]
    hy = [torch.empty(T, d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dx = [torch.empty(T, d, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    hb = [layers[r][2].cpu().pin_memory() if layers[r][2] is not None else None for r in range(R)]
    db = [torch.empty_like(layers[0][2]) for _ in range(2)] if layers[0][2] is not None else None
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    ev_in, ev_out, ev_cp = [ev() for _ in range(steps)], [ev() for _ in range(steps)], [ev() for _ in range(steps)]
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    h2d = T * d * 2 + (hb[0].numel() if hb[0] is not None else 0)
    start.record(h2d_s)
    for i in range(steps):
        s = i % 2
        with torch.cuda.stream(h2d_s):  # x of step i into slot s, once step i-2 has consumed it
            if i >= 2:
                h2d_s.wait_event(ev_out[i - 2])
            dx[s].copy_(hx[i % R], non_blocking=True)
            if db is not None:
                db[s].copy_(hb[i % R], non_blocking=True)
            ev_in[i].record(h2d_s)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[i])
            if i >= R:  # this instance's y of step i-R has been copied out
                stream.wait_event(ev_cp[i - R])
            y = layers[i % R][0].forward(dx[s], bits=None if db is None else db[s], stream=stream)
            ev_out[i].record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(ev_out[i])
            hy[s].copy_(y, non_blocking=True)
            ev_cp[i].record(d2h_s)
    d2h_s.wait_event(ev_out[steps - 1])
    end.record(d2h_s)
    torch.cuda.synchronize()
    return start.elapsed_time(end), h2d, T * d * 2


def instances_for(shape, min_bytes=3 * 126 * 2 ** 20):
    """Layer instances to rotate so that the expert weights of one pass over
    all of them exceed three times the 126 MB L2 (at least 2)."""
    from quantized_moe_expert_histogram_b200 import moeq
    per = shape.E * moeq.moe_blob_bytes(shape.d, shape.F, shape.group, 1 if shape.layout == "planes" else 0)
    return max(2, -(-min_bytes // per))


def measure_workload(name, T, peaks, stream, reps=8):
    """Step time and FFN roofline fraction of another configured workload
    (CUDA graphs over rotated instances, as for the default workload).
    'nested_gate' is the nested-plane layer with its widths chosen on the
    device by the bit-width gate (moe_bit_gate inside the step)."""
    import torch
    from quantized_moe_expert_histogram_b200 import inputs as I
    gate = name == "nested_gate"
    shape = I.SHAPES["nested" if gate else name]
    R = instances_for(shape)
    ls = make_instances(shape, T, R, seed=31, device="cuda", bit_gate=gate)
    ga, gf = capture(ls, stream, "all"), capture(ls, stream, "ffn")
    tot = time_graph(ga, reps, 2, stream) / (reps * R)
    fm = time_graph(gf, reps, 1, stream) / (reps * R)
    b, fl = algorithmic(shape, T, ls[-1][0], shape.layout == "planes")
    tc_bound = fl / (peaks["tc"] * 1e12) > b / (peaks["hbm"] * 1e9)
    out = {"workload": f"{name}: d={shape.d} E={shape.E} top-{shape.k} d_ff={shape.F} "
                       f"{'nested 2/3/4-bit planes' if shape.layout == 'planes' else 'INT4'} g{shape.group}"
                       + (", widths from the bit-width gate" if gate else ""),
           "tokens": T, "instances": R, "tokens_per_s": T / (tot / 1e3), "ms_per_step": tot, "ffn_ms": fm,
           "ffn_bound": "tensor" if tc_bound else "hbm",
           "ffn_frac": (fl / (fm / 1e3) / 1e12 / peaks["tc"]) if tc_bound else (b / (fm / 1e3) / 1e9 / peaks["hbm"]),
           "ffn_alg_bytes": b, "ffn_flops": fl, "launches_per_step": kernel_launches(shape, T, gate)}
    del ls, ga, gf
    torch.cuda.empty_cache()
    return out


def h2d_peak_gbs(nbytes=256 << 20, reps=5):
    """Pinned host -> device copy bandwidth (one large cudaMemcpyAsync)."""
    import torch
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dv = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dv.copy_(h, non_blocking=True)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        for _ in range(reps):
            dv.copy_(h, non_blocking=True)
        b.record(s)
    torch.cuda.synchronize()
    return nbytes * reps / (a.elapsed_time(b) / 1e3) / 1e9


def _time_offload(stack, trace, xs, steps, warm, batch, peak):
    """Time decode steps of an offload stack in its current schedule: wall
    clock around whole steps, copy and compute busy times from CUDA events
    that exclude each stream's waits for the other, giving
        overlap = (copy + compute - wall) / min(copy, compute)
    (1 = the shorter of the two is hidden entirely, 0 = none of it)."""
    import torch
    stack.prefetched = 0
    for s in range(warm):
        stack.step(xs[s], trace[s])
    torch.cuda.synchronize()
    stack.timing(True)
    hits = misses = nbytes = 0
    t0 = time.perf_counter()
    for s in range(warm, warm + steps):
        _, st = stack.step(xs[s], trace[s])
        for h, m, b, _w in st:
            hits, misses, nbytes = hits + h, misses + m, nbytes + b
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    copy_ms, comp_ms = stack.timing_read()
    stack.timing(False)
    wall_ms = wall * 1e3
    h2d = nbytes / wall / 1e9
    return {"tokens_per_s": batch * steps / wall, "ms_per_step": wall_ms / steps,
            "h2d_bytes_per_step": nbytes / steps, "h2d_gbs": h2d, "h2d_frac": h2d / peak,
            "hit_rate": hits / max(1, hits + misses),
            "copy_busy_ms_per_step": copy_ms / steps, "compute_busy_ms_per_step": comp_ms / steps,
            "overlap": (copy_ms + comp_ms - wall_ms) / max(1e-9, min(copy_ms, comp_ms)),
            "prefetch_copies_per_step": stack.prefetched / (warm + steps)}


def run_offload(steps, layers=16, slots=16, batch=8, seed=0, warm=16):
    """The offload workload: stacked OLMoE-shaped layers with experts in pinned
    host memory and a slot cache per layer, decode steps at a fixed batch on a
    Zipf + successor-correlated routing trace, in three schedules on the same
    stack: a routed-id sync per layer ("sync"), that plus predictive
    prefetching of the next layer's experts ("prefetch"), and lookahead
    (every layer's ids known at the start of the step, one id copy per step,
    no per-layer sync).  Timing as in _time_offload."""
    import torch
    from quantized_moe_expert_histogram_b200 import inputs as I
    from quantized_moe_expert_histogram_b200.offload import OffloadStack
    shape = I.SHAPES["olmoe"]
    stack = OffloadStack(shape, layers, slots, batch, seed=seed, prefetch=True)
    n = steps + warm
    trace = I.make_slot_trace(shape.E, shape.k, layers, n, batch, seed=seed + 1).cuda()
    xs = I.make_slot_x(shape.d, n, batch, seed=seed + 1, device="cuda")
    peak = h2d_peak_gbs()
    out = {"workload": f"{layers} OLMoE-shaped layers (d=2048, E=64, top-8, d_ff=1024, INT4 g128), "
                       f"{slots} GPU slots per layer, batch {batch}, Zipf routing with 70% successor correlation",
           "steps": steps, "warmup_steps": warm, "h2d_peak_gbs": peak,
           "timing": "host wall clock around whole steps; copy/compute busy time from CUDA events"}
    for mode in ("sync", "prefetch", "lookahead"):
        stack.prefetch, stack.lookahead = mode == "prefetch", mode == "lookahead"
        out[mode] = _time_offload(stack, trace, xs, steps, warm, batch, peak)
    stack.close()
    return out


def run_offload_nested(steps, layers=8, slots=8, batch=4, seed=0, warm=16):
    """The nested-plane offload workload: stacked nested 2/3/4-bit layers
    (d=4096, E=16, top-4, d_ff=1024, g128), each with a bit-width gate that
    picks every assignment's width, experts in pinned host memory, on the
    same kind of routing trace.  Each schedule (per-layer sync, lookahead)
    runs once with plane-mode caches (only the planes up to the widths used
    are copied, missing planes added on upgrade) and once with whole-blob
    caches over the same host blobs."""
    import torch
    from quantized_moe_expert_histogram_b200 import inputs as I
    from quantized_moe_expert_histogram_b200.offload import OffloadStack
    shape = I.SHAPES["nested"]
    stack = OffloadStack(shape, layers, slots, batch, seed=seed)
    n = steps + warm
    trace = I.make_slot_trace(shape.E, shape.k, layers, n, batch, seed=seed + 2).cuda()
    xs = I.make_slot_x(shape.d, n, batch, seed=seed + 2, device="cuda")
    peak = h2d_peak_gbs()
    out = {"workload": f"{layers} nested-plane layers (d=4096, E=16, top-4, d_ff=1024, planes 2+1+1 g128), "
                       f"widths from a bit-width gate per layer, {slots} GPU slots per layer, batch {batch}, "
                       f"Zipf routing with 70% successor correlation",
           "blob_bytes": stack.blob_bytes, "steps": steps, "warmup_steps": warm, "h2d_peak_gbs": peak}
    for mode in ("sync", "lookahead"):
        stack.lookahead = mode == "lookahead"
        for planes in (True, False):
            stack.set_plane_staging(planes)
            out[f"{mode}_{'planes' if planes else 'whole'}"] = _time_offload(stack, trace, xs, steps, warm,
                                                                              batch, peak)
    stack.close()
    return out


def cpu_baseline(shape, T, seed, sample_tokens, budget_s=20.0):
    """The oracle as it stands, on the host cores, on a bounded token sample."""
    import numpy as np
    import torch
    from oracle import moe_oracle as O
    from quantized_moe_expert_histogram_b200 import inputs as I
    L = I.make_layer(shape, T, seed=seed, device="cpu")
    x = L["x"].float().numpy()
    bias = L["bias"].numpy() if L["bias"] is not None else None
    bits = L["bits"].numpy() if "bits" in L else None
    ex = O.QuantExperts(L["w_gate"].numpy(), L["w_up"].numpy(), L["w_down"].numpy(), shape.group)
    n = sample_tokens or min(T, 64)
    sub = np.arange(n)
    # offline quantisation of the experts the sample needs is not part of a step
    out = O.moe_layer(x, L["w_router"].numpy(), bias, shape.k, ex, bits=bits, token_subset=sub[:1])
    need = set(out["sel"][:n].reshape(-1).tolist())
    for e in need:
        ex.quant(int(e))
    t0 = time.perf_counter()
    reps = 0
    while True:
        O.moe_layer(x[:n], L["w_router"].numpy(), bias, shape.k, ex,
                    bits=None if bits is None else bits[:n])
        reps += 1
        if time.perf_counter() - t0 > budget_s or reps >= 3:
            break
    dt = time.perf_counter() - t0
    cores = os.cpu_count()
    return {"value": n * reps / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} of the {T} tokens (route, permute, FFN, combine of the sample), x{reps}, "
                      f"fp64 numpy oracle; expert quantisation done beforehand"}


# ------------------------------------------------------------------ main --

def run_reference(args):
    world, rank, _ = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0
    if rank != 0:
        return
    from quantized_moe_expert_histogram_b200 import inputs as I
    shape = I.SHAPES[args.workload]
    T = args.tokens
    per_step = []
    cb = None
    n = args.cpu_sample_tokens or 32
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(shape, T, 0, n, budget_s=0.0)  # one pass over the sample per step
        if i >= args.warmup:
            per_step.append(cb["value"])
    v = statistics.mean(per_step)
    cb["value"] = v
    ms = statistics.mean(1000.0 * n / x for x in per_step)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{shape.name} MoE layer d={shape.d} E={shape.E} top-{shape.k} "
                                   f"d_ff={shape.F} INT4 g{shape.group}", "tokens": T},
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    from quantized_moe_expert_histogram_b200 import build as B
    from quantized_moe_expert_histogram_b200 import inputs as I
    from quantized_moe_expert_histogram_b200 import moeq
    B.build()
    world, rank, local = dist_setup(args)
    moeq.load()
    gate = args.workload == "nested_gate"  # nested layer, widths from the bit gate
    shape = I.SHAPES["nested" if gate else args.workload]
    T = args.tokens
    peaks = load_peaks()
    stream = torch.cuda.Stream()
    if args.profile:
        layers = make_instances(shape, T, 1, seed=0, device="cuda", bit_gate=gate)
        for _ in range(args.warmup + args.steps):
            _step_calls(*layers[0], stream, "all")
        torch.cuda.synchronize()
        print(f"profile run done: {shape.name} T={T} steps={args.warmup + args.steps}")
        return
    layers = make_instances(shape, T, args.instances, seed=rank * 7919, device="cuda", bit_gate=gate)
    torch.cuda.synchronize()

    R = len(layers)
    replays = max(1, (args.steps + R - 1) // R)
    steps = replays * R
    g_all = capture(layers, stream, "all")
    g_ffn = capture(layers, stream, "ffn")
    barrier(world)
    clocks = ClockSampler(local)
    clocks.start()
    torch.cuda.synchronize()
    total_ms = time_graph(g_all, replays, max(1, args.warmup // R + 1), stream)
    clk = clocks.stop()
    ffn_total = time_graph(g_ffn, replays, 1, stream)
    ffn_ms = ffn_total / steps
    barrier(world)
    total_ms = max_over_ranks(world, total_ms)
    ms_per_step = total_ms / steps
    value = job_throughput(world, T, steps, total_ms)
    del g_all, g_ffn

    bytes_alg, flops = algorithmic(shape, T, layers[-1][0], layers[0][2] is not None)
    t_ffn = ffn_ms / 1e3
    tc_bound = flops / (peaks["tc"] * 1e12) > bytes_alg / (peaks["hbm"] * 1e9)
    if tc_bound:
        peak = peaks["tc_sust"] if total_ms > 1000 else peaks["tc"]
        ach = flops / t_ffn / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak}
    else:
        ach = bytes_alg / t_ffn / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s", "frac": ach / peaks["hbm"]}
    traffic, traffic_src = profiled_traffic(shape.name, T)
    roof.update({"traffic": traffic, "traffic_source": traffic_src,
                 "kernel": "moe_grouped_ffn_wq (gate/up + down launches)",
                 "timing": "FFN-only CUDA graph over the same rotated instances, events around the replays",
                 "peak_source": peaks["src"], "ffn_ms": ffn_ms,
                 "per_launch_units": f"{T * shape.k} assignments"})

    e2e_ms, h2d, d2h = time_e2e(layers, steps, stream)
    e2e_ms = max_over_ranks(world, e2e_ms)
    e2e = {"value": job_throughput(world, T, steps, e2e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    sweep = {}
    for tok in [int(x) for x in args.sweep.split(",") if x.strip()]:
        ls = make_instances(shape, tok, 16, seed=rank * 7919 + 17, device="cuda")
        ga, gf = capture(ls, stream, "all"), capture(ls, stream, "ffn")
        rep = max(4, 64 // len(ls))
        tot = time_graph(ga, rep, 2, stream) / (rep * len(ls))
        fm = time_graph(gf, rep, 1, stream) / (rep * len(ls))
        b, fl = algorithmic(shape, tok, ls[-1][0], ls[0][2] is not None)
        sweep[str(tok)] = {"tokens_per_s": tok / (tot / 1e3), "ms_per_step": tot, "ffn_ms": fm,
                           "ffn_hbm_frac": b / (fm / 1e3) / 1e9 / peaks["hbm"],
                           "ffn_tc_frac": fl / (fm / 1e3) / 1e12 / peaks["tc"]}
        del ls, ga, gf
        torch.cuda.empty_cache()

    workloads = []
    if args.workloads:
        for item in args.workloads.split(","):
            name, tok = item.split(":")
            workloads.append(measure_workload(name, int(tok), peaks, stream))

    offload = None
    if world == 1 and args.offload_steps > 0:
        del layers
        torch.cuda.empty_cache()
        offload = run_offload(args.offload_steps)
        offload["nested"] = run_offload_nested(max(1, args.offload_steps // 4))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(shape, T, 0, args.cpu_sample_tokens)

    # our kernels per step: router 2, permutation 1 + gather (<= 1024 assignments) or
    # 3 + gather, FFN 2, combine 1
    launches_per_step = kernel_launches(shape, T)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp16", "data": "synthetic",
            "config": {"workload": f"{shape.name} MoE layer d={shape.d} E={shape.E} top-{shape.k} "
                                   f"d_ff={shape.F} INT4 g{shape.group}", "tokens": T,
                       "global_batch": T * world, "parallelism": f"replicas x{world}",
                       "l2": f"{args.instances} layer instances rotated ({shape.E} experts x "
                             f"{moeq.moe_blob_bytes(shape.d, shape.F, shape.group, 0)} B each), inputs > L2"},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * steps,
            "clocks": clk, "sweep": sweep, "workloads": workloads, "offload": offload}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
