"""Throughput bench of the bifocal hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  * prefill of the Qwen3-8B-shaped layer at 128K (batch 1, 32 q heads / 8 kv
    heads, head_dim 128, RoPE base 1e6, L 131072, w_pretrained 32768 -> G 4,
    w0 4096) through the default path (the one held to the oracle's
    tolerances on every workload): the key-row correction pass, then the fused
    tcgen05 kernel that corrects the query block itself and carries remote
    scores as fp16 hi + lo products;
  * decode of the Qwen3-4B-shaped layer at 128K (32 / 8 heads, head_dim 128,
    batch 8, cache of 131072 base-rotated keys, G 4, w0 4096).
`value` is the prefill TFLOP/s (algorithmic 4 * B * Hq * d * L(L+1)/2 per
step, summed over ranks, divided by the max-over-ranks device time of the
prefill calls); the decode GB/s (K and V bytes read once) is reported beside
it, and so are the other prefill paths (single fp16 product, key tiles
corrected inside the kernel, the three-call inclusion-exclusion formulation,
plain RoPE), the Qwen3-1.7B 64K and tiny workloads, the length / band sweep,
varlen decode, the new-token append and chunked prefill.  Inputs are larger
than L2 (1 GiB Q, 4 GiB KV cache), so no flush runs between steps.

  python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]

For N > 1 launch under torch.distributed.run; every rank runs its own
independent sequences (weak scaling, no data-path collective).
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

METRIC = "bifocal prefill TFLOP/s @128K; decode HBM GB/s @128K; % of B200 roofline"

PREFILL = dict(workload="qwen3-8b-shaped bifocal prefill, single layer", B=1, L=131072, Hq=32, Hkv=8, D=128,
               W=32768, w0=4096, base=1e6)
DECODE = dict(workload="qwen3-4b-shaped bifocal decode", B=8, L=131072, Hq=32, Hkv=8, D=128, W=32768, w0=4096,
              base=1e6)
# the other workloads of the method's evaluation shapes, reported beside the headline
PREFILL_1P7B = dict(workload="qwen3-1.7b-shaped bifocal prefill, single layer", B=1, L=65536, Hq=16, Hkv=8, D=128,
                    W=32768, w0=4096, base=1e6)
PREFILL_TINY = dict(workload="tiny bifocal prefill", B=1, L=512, Hq=2, Hkv=1, D=64, W=128, w0=32, base=1e4)
SWEEP_L = (16384, 32768, 32769, 49152, 100003, 131072)  # qwen3-4b shape, w0 in {0, 4096, L}, 1% x8 key outliers

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def prefill_flop(c):
    return 4.0 * c["B"] * c["Hq"] * c["D"] * c["L"] * (c["L"] + 1) / 2.0


def decode_bytes(c):
    return 2.0 * c["B"] * c["L"] * c["Hkv"] * c["D"] * 2.0


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Source files that determine each timed kernel's code and launch shape; a
# traffic figure is used only while these hash to the value stored with it.
KERNEL_SOURCES = {
    "prefill_attention": ["prefill_hilo_sm100.cu", "jl_common.cuh", "jl_kernels.cuh", "jl_api.cu"],
    "decode": ["decode_sm100.cu", "jl_common.cuh", "jl_kernels.cuh", "jl_api.cu"],
}


def load_traffic():
    """Per-launch DRAM bytes of the timed kernels from the committed ncu summary,
    each valid only while its kernel's sources hash to the value recorded with it."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return {}
    try:
        with open(path) as f:
            data = json.load(f)
    except (OSError, ValueError):
        return {}
    return {k: v for k, v in data.items()
            if isinstance(v, dict) and k in KERNEL_SOURCES and v.get("sources") == sources_hash(KERNEL_SOURCES[k])}


def sources_hash(files):
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rope_context_extension_b200", "csrc")
    for name in sorted(files):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled every 20 ms
    through NVML while the timed region runs (nvidia-smi at 200 ms when NVML
    is not importable).  Only samples taken between mark_begin() and
    mark_end() count, so the median is the clock under load."""

    # NVML clock-event reason bits
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80}
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, torch_device: int):
        self.dev = torch_device
        self.samples = []  # (time, sm_mhz, power_w, reasons)
        self.window = [None, None]
        self.stop_evt = threading.Event()
        self.thread = None
        self.proc = None
        self.nvml = None
        self.handle = None
        self.smax = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        self.nvml = pynvml
        uuid = str(getattr(torch.cuda.get_device_properties(self.dev), "uuid", "") or "")
        if uuid:
            try:
                return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        idx = int(vis.split(",")[self.dev]) if vis and vis.split(",")[0].isdigit() else self.dev
        return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def start(self):
        try:
            self.handle = self._nvml_handle()
            nv = self.nvml
            self.smax = float(nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons

            def loop():
                while not self.stop_evt.is_set():
                    t = time.perf_counter()
                    try:
                        sm = float(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                        pw = nv.nvmlDeviceGetPowerUsage(self.handle) / 1e3
                        rs = int(get_reasons(self.handle))
                    except Exception:
                        break
                    self.samples.append((t, sm, pw, rs))
                    self.stop_evt.wait(0.02)
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.handle = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()

    def _read_smi(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, self.smax = float(parts[1]), float(parts[2])
                pw = float(parts[3])
            except ValueError:
                continue
            rs = 0
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    rs |= self.REASONS[n]
            self.samples.append((time.perf_counter(), sm, pw, rs))

    def mark_begin(self):
        self.window[0] = time.perf_counter()

    def mark_end(self):
        self.window[1] = time.perf_counter()

    def stop(self):
        self.stop_evt.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        if self.handle is None and self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no NVML and no nvidia-smi"]}
        return self.summarize(self.samples, self.window, self.smax,
                              "nvml 20 ms" if self.handle is not None else "nvidia-smi 200 ms")

    @classmethod
    def summarize(cls, samples, window, smax, source):
        """Clock summary of the samples (time, sm_mhz, power_w, reason bits)
        taken inside window = [begin, end] (either may be None: unbounded)."""
        t0 = window[0] if window[0] is not None else -math.inf
        t1 = window[1] if window[1] is not None else math.inf
        inside = [x for x in samples if t0 <= x[0] <= t1]
        reasons = sorted(n for n, bit in cls.REASONS.items() if any(x[3] & bit for x in inside))
        return {"sm_mhz": statistics.median(x[1] for x in inside) if inside else None, "sm_max_mhz": smax,
                "sm_mhz_min": min(x[1] for x in inside) if inside else None,
                "power_w_median": round(statistics.median(x[2] for x in inside), 1) if inside else None,
                "reasons": reasons, "samples": len(inside), "source": source}


def dist_setup(n_gpus):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a per-rank timing over all ranks (the only collective the bench
    makes; no data-path exchange)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank, world, max_ms):
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank / (max_ms * 1e-3)


def gen_on_device(shape, seed, dev):
    import torch
    g = torch.Generator(device=dev).manual_seed(seed)
    return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)


def scale_outliers_on_device(k, frac, seed, scale=8.0):
    """Multiply a seeded `frac` share of the (b, j, kv-head) rows of k by `scale`."""
    import torch
    B, L, H, _ = k.shape
    g = torch.Generator(device=k.device).manual_seed(seed)
    n = max(1, int(round(frac * B * L * H)))
    idx = torch.randperm(B * L * H, generator=g, device=k.device)[:n]
    kf = k.view(B * L * H, -1)
    kf[idx] = (kf[idx].float() * scale).to(torch.bfloat16)
    return k


def executed_prefill_flop(c, jl):
    """Flop the tensor core executes for one prefill of workload c on the
    default path: one 128 x 128 tile product (S or P V) is 2 * 128 * 128 * D
    flop; a local pass issues S once, a remote pass three times (hi + lo),
    and every pass issues one P V.  Diagnostic beside the algorithmic count."""
    loc_only, both, rem_only, _ = jl.jl_prefill_tile_classes(c["L"], c["w0"], c["W"])
    per_tile = 2.0 * 128 * 128 * c["D"]
    G = jl.jl_group_size(c["L"], c["W"])
    if G == 1 or c["w0"] >= c["L"]:
        units = 2.0 * (loc_only + both + rem_only)
    else:
        units = 2.0 * (loc_only + both) + 4.0 * (rem_only + both)
    return per_tile * units * c["B"] * c["Hq"]


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def bench_config(world):
    """The workload description both arms print (the reference arm times the
    oracle on the prefill part of it)."""
    P, Dc = PREFILL, DECODE
    return {
        "workload": P["workload"] + " + " + Dc["workload"],
        "prefill": {k_: P[k_] for k_ in ("B", "L", "Hq", "Hkv", "D", "W", "w0", "base")},
        "decode": {k_: Dc[k_] for k_ in ("B", "L", "Hq", "Hkv", "D", "W", "w0", "base")},
        "query_shift": "self_extend",
        "l2": "inputs larger than L2",
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
    }


def run_ours(args):
    import torch
    from rope_context_extension_b200 import jetlong as jl

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    P, Dc = PREFILL, DECODE
    seed = 1000 * rank
    SE = jl.JL_QSHIFT_SELF_EXTEND

    # prefill buffers (resident in HBM)
    q = gen_on_device((P["B"], P["L"], P["Hq"], P["D"]), seed + 0, dev)
    k = gen_on_device((P["B"], P["L"], P["Hkv"], P["D"]), seed + 1, dev)
    v = gen_on_device((P["B"], P["L"], P["Hkv"], P["D"]), seed + 2, dev)
    o = torch.empty_like(q)
    lse = torch.empty(P["B"], P["Hq"], P["L"], dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(jl.jl_prefill_workspace_bytes(P["B"], P["L"], P["Hq"], P["Hkv"], P["D"]), dtype=torch.uint8,
                     device=dev)
    # decode buffers
    dq = gen_on_device((Dc["B"], Dc["Hq"], Dc["D"]), seed + 3, dev)
    kc = gen_on_device((Dc["B"], Dc["L"], Dc["Hkv"], Dc["D"]), seed + 4, dev)
    vc = gen_on_device((Dc["B"], Dc["L"], Dc["Hkv"], Dc["D"]), seed + 5, dev)
    do = torch.empty_like(dq)
    dlse = torch.empty(Dc["B"], Dc["Hq"], dtype=torch.float32, device=dev)
    dws = torch.zeros(jl.jl_decode_workspace_bytes(Dc["B"], Dc["L"], Dc["Hq"], Dc["Hkv"], Dc["D"]),
                      dtype=torch.uint8, device=dev)

    def prefill_step(evs=None, w0=None, mode=SE, wsp=ws):
        # stage 1: the correction pass (the key rows' hi / lo parts); stage 2:
        # the attention kernel
        w = P["w0"] if w0 is None else w0
        if evs:
            evs[0].record(stream)
        jl.jl_prefill_correction(q, k, w0=w, w_pretrained=P["W"], rope_base=P["base"], mode=mode, workspace=wsp,
                                 dev_error=err, stream=stream)
        if evs:
            evs[1].record(stream)
        jl.jl_prefill_attention(q, k, v, o, lse, w0=w, w_pretrained=P["W"], rope_base=P["base"], mode=mode,
                                workspace=wsp, dev_error=err, stream=stream)
        if evs:
            evs[2].record(stream)

    def decode_step(evs=None, w0=None):
        w = Dc["w0"] if w0 is None else w0
        if evs:
            evs[0].record(stream)
        jl.jl_bifocal_decode(dq, kc, vc, do, dlse, L=Dc["L"], w0=w, w_pretrained=Dc["W"], rope_base=Dc["base"],
                             workspace=dws, dev_error=err, stream=stream)
        if evs:
            evs[1].record(stream)

    for _ in range(args.warmup):
        prefill_step()
        decode_step()
    torch.cuda.synchronize()

    K = args.steps
    pev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    dev_ = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark_begin()
    t0.record(stream)
    for i in range(K):
        prefill_step(pev[i])
        decode_step(dev_[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    barrier(world)
    clk = clocks.stop()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error {int(err.item())} during the timed region")

    total_ms = t0.elapsed_time(t1)
    corr_ms = sum(e[0].elapsed_time(e[1]) for e in pev) / K
    attn_ms = sum(e[1].elapsed_time(e[2]) for e in pev) / K
    dec_ms = sum(e[0].elapsed_time(e[1]) for e in dev_) / K
    pre_ms = corr_ms + attn_ms
    total_ms = max_over_ranks(total_ms, world)
    pre_ms_max = max_over_ranks(pre_ms, world)
    attn_ms_max = max_over_ranks(attn_ms, world)
    dec_ms_max = max_over_ranks(dec_ms, world)

    flop = prefill_flop(P)
    dbytes = decode_bytes(Dc)
    value = weak_scaling_value(flop, world, pre_ms_max) / 1e12
    attn_tflops = flop / (attn_ms_max * 1e-3) / 1e12
    dec_gbs_kernel = dbytes / (dec_ms_max * 1e-3) / 1e9
    exec_flop = executed_prefill_flop(P, jl)

    def time_calls(fn, reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fn()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    # decode on its own, launches back to back as a serving loop issues them
    # (the in-step decode above runs right after the prefill, under its power
    # cap); B 8 and B 1 against the same 128K cache
    def decode_loop(bsz, seconds=0.6):
        qb, kb, vb, ob, lb = dq[:bsz], kc[:bsz], vc[:bsz], do[:bsz], dlse[:bsz]

        def call():
            jl.jl_bifocal_decode(qb, kb, vb, ob, lb, L=Dc["L"], w0=Dc["w0"], w_pretrained=Dc["W"],
                                 rope_base=Dc["base"], workspace=dws, dev_error=err, stream=stream)
        for _ in range(5):
            call()
        cal = time_calls(call, 10)
        reps = int(max(20, min(5000, seconds * 1e3 / max(cal, 1e-3))))
        sampler = ClockSampler(local)
        sampler.start()
        time.sleep(0.3)
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        sampler.mark_begin()
        a_.record(stream)
        for _ in range(reps):
            call()
        b_.record(stream)
        torch.cuda.synchronize()
        sampler.mark_end()
        barrier(world)
        clk_ = sampler.stop()
        ms = max_over_ranks(a_.elapsed_time(b_) / reps, world)
        by = decode_bytes(dict(Dc, B=bsz))
        return {"B": bsz, "ms": round(ms, 4), "gbs": round(by / (ms * 1e-3) / 1e9, 1),
                "gbs_all_ranks": round(weak_scaling_value(by, world, ms) / 1e9, 1),
                "tokens_per_s": round(world * bsz / (ms * 1e-3), 1), "reps": reps, "clocks": clk_}

    if args.no_decode_loops:
        dloop8 = dloop1 = {"B": 0, "ms": dec_ms_max, "gbs": round(dec_gbs_kernel, 1), "reps": 0, "clocks": None,
                           "gbs_all_ranks": round(weak_scaling_value(dbytes, world, dec_ms_max) / 1e9, 1),
                           "tokens_per_s": round(world * Dc["B"] / (dec_ms_max * 1e-3), 1)}
    else:
        dloop8 = decode_loop(Dc["B"])
        dloop1 = decode_loop(1)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error {int(err.item())} during the decode loops")

    # plain causal RoPE from the same library entry points (w0 = L)
    plain_pre_ms = time_calls(lambda: prefill_step(w0=P["L"]), max(2, K // 2))
    plain_dec_ms = time_calls(lambda: decode_step(w0=Dc["L"]), max(2, K // 2))
    # the other prefill paths on the same inputs
    paths = {}
    for name, flag in (("fp16_single_product", jl.JL_PREFILL_FP16),
                       ("keys_corrected_in_kernel", jl.JL_PREFILL_KEYS_IN_KERNEL)):
        if args.no_variants:
            break
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ms = time_calls(lambda: prefill_step(mode=SE | flag), 2)
        prefill_step(evs, mode=SE | flag)
        torch.cuda.synchronize()
        paths[name] = {"ms": round(ms, 3), "tflops": round(flop / (ms * 1e-3) / 1e12, 2),
                       "correction_ms": round(evs[0].elapsed_time(evs[1]), 3),
                       "attention_ms": round(evs[1].elapsed_time(evs[2]), 3),
                       "speed_vs_default": round(pre_ms_max / ms, 3)}
    ie = None
    if not args.no_ie:
        ws3 = torch.empty(jl.jl_prefill_ie_workspace_bytes(P["B"], P["L"], P["Hq"], P["Hkv"], P["D"]),
                          dtype=torch.uint8, device=dev)
        ie_ms = time_calls(lambda: jl.jl_bifocal_prefill_ie(q, k, v, o, lse, w0=P["w0"], w_pretrained=P["W"],
                                                            rope_base=P["base"], workspace=ws3, dev_error=err,
                                                            stream=stream), 2)
        ie = {"ms": round(ie_ms, 3), "tflops": round(flop / (ie_ms * 1e-3) / 1e12, 2),
              "fused_speedup": round(ie_ms / pre_ms_max, 3)}
        del ws3
    if int(err.item()) != 0:
        raise RuntimeError(f"device error {int(err.item())} in the prefill variants")

    # the other workloads: Qwen3-1.7B 64K and tiny prefill (bifocal and plain),
    # and the length / band sweep (prefill and B 1 decode, 1% x8 key outliers)
    others = None
    if not args.no_other_workloads:
        others = {}
        for c in (PREFILL_1P7B, PREFILL_TINY):
            q2 = gen_on_device((c["B"], c["L"], c["Hq"], c["D"]), seed + 11, dev)
            k2 = gen_on_device((c["B"], c["L"], c["Hkv"], c["D"]), seed + 12, dev)
            v2 = gen_on_device((c["B"], c["L"], c["Hkv"], c["D"]), seed + 13, dev)
            o2 = torch.empty_like(q2)
            l2 = torch.empty(c["B"], c["Hq"], c["L"], dtype=torch.float32, device=dev)
            w2 = torch.empty(jl.jl_prefill_workspace_bytes(c["B"], c["L"], c["Hq"], c["Hkv"], c["D"]),
                             dtype=torch.uint8, device=dev)
            res = {}
            for tag, w0 in (("bifocal", c["w0"]), ("plain", c["L"])):
                reps = 3 if c["L"] > 8192 else 200
                ms = time_calls(lambda: jl.jl_bifocal_prefill(q2, k2, v2, o2, l2, w0=w0, w_pretrained=c["W"],
                                                              rope_base=c["base"], workspace=w2, dev_error=err,
                                                              stream=stream), reps)
                f = prefill_flop(c)
                res[tag] = {"ms": round(ms, 4), "tflops": round(f / (ms * 1e-3) / 1e12, 2),
                            "tokens_per_s": round(c["B"] * c["L"] / (ms * 1e-3), 1)}
            res["shape"] = {k_: c[k_] for k_ in ("B", "L", "Hq", "Hkv", "D", "W", "w0", "base")}
            others[c["workload"]] = res
            del q2, k2, v2, o2, l2, w2
        sweep = []
        sh = dict(B=1, Hq=32, Hkv=8, D=128, W=32768, base=1e6)
        dws1 = torch.zeros(jl.jl_decode_workspace_bytes(1, max(SWEEP_L), 32, 8, 128), dtype=torch.uint8, device=dev)
        for L in SWEEP_L:
            q2 = gen_on_device((1, L, 32, 128), seed + L, dev)
            k2 = scale_outliers_on_device(gen_on_device((1, L, 8, 128), seed + L + 1, dev), 0.01, seed + 7)
            v2 = gen_on_device((1, L, 8, 128), seed + L + 2, dev)
            o2 = torch.empty_like(q2)
            l2 = torch.empty(1, 32, L, dtype=torch.float32, device=dev)
            qd1, od1 = q2[:, L - 1].contiguous(), torch.empty(1, 32, 128, dtype=torch.bfloat16, device=dev)
            ld1 = torch.empty(1, 32, dtype=torch.float32, device=dev)
            w2 = torch.empty(jl.jl_prefill_workspace_bytes(1, L, 32, 8, 128), dtype=torch.uint8, device=dev)
            for w0 in (0, 4096, L):
                c = dict(sh, L=L, w0=w0)
                pms = time_calls(lambda: jl.jl_bifocal_prefill(q2, k2, v2, o2, l2, w0=w0, w_pretrained=sh["W"],
                                                               rope_base=sh["base"], workspace=w2, dev_error=err,
                                                               stream=stream), 2)
                dms = time_calls(lambda: jl.jl_bifocal_decode(qd1, k2, v2, od1, ld1, L=L, w0=w0,
                                                              w_pretrained=sh["W"], rope_base=sh["base"],
                                                              workspace=dws1, dev_error=err, stream=stream), 20)
                sweep.append({"L": L, "w0": w0, "G": jl.jl_group_size(L, sh["W"]),
                              "prefill_ms": round(pms, 3), "prefill_tflops": round(prefill_flop(c) / (pms * 1e-3) / 1e12, 2),
                              "prefill_tokens_per_s": round(L / (pms * 1e-3), 1),
                              "decode_ms": round(dms, 4), "decode_gbs": round(decode_bytes(c) / (dms * 1e-3) / 1e9, 1),
                              "decode_tokens_per_s": round(1 / (dms * 1e-3), 1)})
            del q2, k2, v2, o2, l2, w2
        others["length / band sweep (qwen3-4b shape, 1% x8 key outliers, decode B 1)"] = sweep
        del dws1

        # varlen decode: one batch of the decode workload's cache whose
        # sequences have lengths across the group sizes G = 1 .. 4 (the cache
        # is read up to each sequence's own length)
        Lm, Wd = Dc["L"], Dc["W"]
        lens = [Lm // 8, Lm // 4, Lm // 4 + 1, 3 * Lm // 8, Lm // 2 + 1, 3 * Lm // 4, Lm, Lm][:Dc["B"]]
        sl = torch.tensor(lens, dtype=torch.int32, device=dev)
        bsz = len(lens)
        vms = time_calls(lambda: jl.jl_bifocal_decode_varlen(dq[:bsz], kc[:bsz], vc[:bsz], do[:bsz], dlse[:bsz], sl,
                                                             max_len=Lm, w0=Dc["w0"], w_pretrained=Wd,
                                                             rope_base=Dc["base"], workspace=dws, dev_error=err,
                                                             stream=stream), 200)
        vbytes = sum(2.0 * L_ * Dc["Hkv"] * Dc["D"] * 2.0 for L_ in lens)
        hbm = load_peaks()[0]["hbm_gbs"]
        others["varlen decode (qwen3-4b shape, mixed lengths)"] = {
            "lengths": lens, "G": [jl.jl_group_size(L_, Wd) for L_ in lens], "ms": round(vms, 4),
            "gbs": round(vbytes / (vms * 1e-3) / 1e9, 1), "frac": round(vbytes / (vms * 1e-3) / 1e9 / hbm, 4),
            "tokens_per_s": round(bsz / (vms * 1e-3), 1)}
        # the new-token append: rotate each sequence's new q and k at its
        # position and write k, v into that cache row (the row after each
        # length above, or the last row of a full cache; timed after the
        # varlen call, which therefore read the cache unchanged)
        qn = gen_on_device((bsz, Dc["Hq"], Dc["D"]), seed + 21, dev)
        kn = gen_on_device((bsz, Dc["Hkv"], Dc["D"]), seed + 22, dev)
        vn = gen_on_device((bsz, Dc["Hkv"], Dc["D"]), seed + 23, dev)
        qo = torch.empty_like(qn)
        pos = torch.tensor([min(L_, Lm - 1) for L_ in lens], dtype=torch.int32, device=dev)
        ams = time_calls(lambda: jl.jl_rope_append(qn, kn, vn, pos, qo, kc[:bsz], vc[:bsz], rope_base=Dc["base"],
                                                   dev_error=err, stream=stream), 1000)
        others["new-token append (qwen3-4b shape, one token per sequence)"] = {
            "B": bsz, "us": round(ams * 1e3, 2), "tokens_per_s": round(bsz / (ams * 1e-3), 1)}
        del qn, kn, vn, qo
        # chunked prefill: the prefill workload's last chunk of queries against
        # its cache (the keys of every earlier position already there)
        C_ = min(8192, P["L"] // 2)
        off = P["L"] - C_
        qc = q[:, off:].contiguous()
        oc = torch.empty_like(qc)
        lc = torch.empty(P["B"], P["Hq"], C_, dtype=torch.float32, device=dev)
        wc = torch.empty(jl.jl_prefill_chunk_workspace_bytes(P["B"], off, C_, P["Hq"], P["Hkv"], P["D"]),
                         dtype=torch.uint8, device=dev)
        cms = time_calls(lambda: jl.jl_bifocal_prefill_chunk(qc, k, v, oc, lc, q_offset=off, w0=P["w0"],
                                                             w_pretrained=P["W"], rope_base=P["base"], workspace=wc,
                                                             dev_error=err, stream=stream), 5)
        cflop = 4.0 * P["B"] * P["Hq"] * P["D"] * (C_ * off + C_ * (C_ + 1) / 2.0)
        others["chunked prefill (qwen3-8b shape, last chunk of the prefill workload)"] = {
            "q_offset": off, "chunk": C_, "ms": round(cms, 3), "tflops": round(cflop / (cms * 1e-3) / 1e12, 2),
            "tokens_per_s": round(P["B"] * C_ / (cms * 1e-3), 1)}
        del qc, oc, lc, wc

        # the multi-GPU decode layouts, one rank's share run alone on this GPU
        # (the collective that follows is not included: the all-gather moves
        # each rank's r x D outputs per head, a few KB): head sharding gives a
        # rank Hkv / world KV heads of every sequence, sequence split gives it
        # L / world keys of every sequence plus the combine of world partials
        from rope_context_extension_b200 import multi_gpu as mg
        layouts = []
        def one_gpu():
            return time_calls(lambda: jl.jl_bifocal_decode(dq, kc, vc, do, dlse, L=Dc["L"], w0=Dc["w0"],
                                                           w_pretrained=Dc["W"], rope_base=Dc["base"], workspace=dws,
                                                           dev_error=err, stream=stream), 100)
        ms1 = one_gpu()
        rank_ms = []
        for world_ in (2, 4, 8):
            entry = {"world": world_}
            if Dc["Hkv"] % world_ == 0:
                kb_, kn_, qb_, qn_ = mg.head_shard_slices(Dc["Hq"], Dc["Hkv"], 0, world_)
                q_r, k_r, v_r = mg.take_heads(dq, qb_, qn_, dim=1), mg.take_heads(kc, kb_, kn_), mg.take_heads(vc, kb_, kn_)
                o_r = torch.empty_like(q_r)
                l_r = torch.empty(Dc["B"], qn_, dtype=torch.float32, device=dev)
                ws_r = torch.zeros(jl.jl_decode_workspace_bytes(Dc["B"], Dc["L"], qn_, kn_, Dc["D"]), dtype=torch.uint8,
                                   device=dev)
                hms = time_calls(lambda: jl.jl_bifocal_decode(q_r, k_r, v_r, o_r, l_r, L=Dc["L"], w0=Dc["w0"],
                                                              w_pretrained=Dc["W"], rope_base=Dc["base"], workspace=ws_r,
                                                              dev_error=err, stream=stream), 100)
                entry["head_shard_rank_ms"] = round(hms, 4)
                rank_ms.append(("head_shard", entry, hms))
                del q_r, k_r, v_r, o_r, l_r, ws_r
            n_ = Dc["L"] // world_
            k_s, v_s = kc[:, :n_].contiguous(), vc[:, :n_].contiguous()
            o_s = torch.empty_like(dq)
            l_s = torch.empty(Dc["B"], Dc["Hq"], dtype=torch.float32, device=dev)
            ws_s = torch.zeros(jl.jl_decode_workspace_bytes(Dc["B"], n_, Dc["Hq"], Dc["Hkv"], Dc["D"]), dtype=torch.uint8,
                               device=dev)
            sms = time_calls(lambda: jl.jl_bifocal_decode_range(dq, k_s, v_s, o_s, l_s, key_offset=0, key_count=n_,
                                                                total_len=Dc["L"], w0=Dc["w0"], w_pretrained=Dc["W"],
                                                                rope_base=Dc["base"], workspace=ws_s, dev_error=err,
                                                                stream=stream), 100)
            o_p = o_s.unsqueeze(0).expand(world_, -1, -1, -1).contiguous()
            l_p = l_s.unsqueeze(0).expand(world_, -1, -1).contiguous()
            cms_ = time_calls(lambda: jl.jl_decode_combine(o_p, l_p, do, dlse, stream=stream), 100)
            entry["sequence_split_rank_ms"] = round(sms, 4)
            entry["sequence_split_combine_ms"] = round(cms_, 4)
            rank_ms.append(("sequence_split", entry, sms + cms_))
            layouts.append(entry)
            del k_s, v_s, o_s, l_s, ws_s, o_p, l_p
        # the one-GPU time before and after the shares (the clock under the
        # power cap drifts between them); the lower one is the reference
        ms1 = min(ms1, one_gpu())
        for name_, entry, t_ in rank_ms:
            entry[name_ + "_speedup_vs_one_gpu"] = round(ms1 / t_, 3)
        others["multi-GPU decode layouts, one rank's share on one GPU (qwen3-4b shape, B 8)"] = {
            "one_gpu_ms": round(ms1, 4), "ranks": layouts,
            "note": "compute share of rank 0 alone; no collective and no second GPU"}
        if int(err.item()) != 0:
            raise RuntimeError(f"device error {int(err.item())} in the other workloads")

    # end to end through the public API: pinned host inputs in, result out, every
    # step.  Pipelined as a serving loop runs it: step i's host-to-device copies
    # (own stream) and step i-1's result copy-back (another stream) overlap the
    # kernels of the neighbouring steps; inputs and outputs are double-buffered
    # on the device.  The serial form (copy in, compute, copy out, one stream)
    # is reported beside it.
    e2e = None
    if not args.no_e2e:
        hq = q.cpu().pin_memory()
        hk = k.cpu().pin_memory()
        hv = v.cpu().pin_memory()
        ho = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for _ in range(2)]
        h_bytes = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2
        d_bytes = ho[0].numel() * 2
        bufs = [(q, k, v, o), (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(o))]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_call(bq, bk, bv, bo):
            jl.jl_bifocal_prefill(bq, bk, bv, bo, lse, w0=P["w0"], w_pretrained=P["W"], rope_base=P["base"],
                                  workspace=ws, dev_error=err, stream=stream)

        def pipelined(reps):
            ev = lambda: torch.cuda.Event()
            in_done = [ev() for _ in range(reps)]
            comp_done = [ev() for _ in range(reps)]
            out_done = [ev() for _ in range(reps)]
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            barrier(world)
            a.record(stream)
            s_in.wait_event(a)
            s_out.wait_event(a)
            for i in range(reps):
                bq, bk, bv, bo = bufs[i % 2]
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])  # the previous user of these inputs is done
                with torch.cuda.stream(s_in):
                    bq.copy_(hq, non_blocking=True)
                    bk.copy_(hk, non_blocking=True)
                    bv.copy_(hv, non_blocking=True)
                in_done[i].record(s_in)
                stream.wait_event(in_done[i])
                if i >= 2:
                    stream.wait_event(out_done[i - 2])  # its output buffer has been read back
                e2e_call(bq, bk, bv, bo)
                comp_done[i].record(stream)
                s_out.wait_event(comp_done[i])
                with torch.cuda.stream(s_out):
                    ho[i % 2].copy_(bo, non_blocking=True)
                out_done[i].record(s_out)
            stream.wait_event(out_done[reps - 1])
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / reps

        def serial(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            barrier(world)
            a.record(stream)
            for _ in range(reps):
                q.copy_(hq, non_blocking=True)
                k.copy_(hk, non_blocking=True)
                v.copy_(hv, non_blocking=True)
                e2e_call(q, k, v, o)
                ho[0].copy_(o, non_blocking=True)
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / reps

        pipelined(2)  # warm-up of the streams and the second buffer set
        e2e_ms = max_over_ranks(pipelined(max(4, K)), world)
        serial_ms = max_over_ranks(serial(max(2, K // 2)), world)
        e2e = {"value": round(world * flop / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h_bytes), "d2h_bytes_per_step": int(d_bytes),
               "ms_per_step": round(e2e_ms, 3), "api": "jl_bifocal_prefill",
               "schedule": "copies on two streams overlapping the neighbouring steps' kernels, double-buffered",
               "serial": {"ms_per_step": round(serial_ms, 3),
                          "value": round(world * flop / (serial_ms * 1e-3) / 1e12, 2)}}
        del bufs
        if int(err.item()) != 0:
            raise RuntimeError(f"device error {int(err.item())} in the end-to-end loop")

    peaks, peak_kind = load_peaks()
    tensor_peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    # the stored traffic figures are per launch of the default (128K) workloads
    traffic = load_traffic() if not (args.prefill_len or args.decode_len or args.decode_batch) else {}
    sm_ghz = (clk.get("sm_mhz") or 0) / 1e3
    peak_ghz = (peaks.get("clocks_under_load", {}).get("sm_mhz_median") or 0) / 1e3
    out = None
    if rank == 0:
        # the oracle's CPU baseline is taken on rank 0 of a one-GPU run only
        cpu = None if (args.no_cpu_baseline or world > 1) else cpu_baseline(seconds=args.cpu_seconds)
        out = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": round(total_ms / K, 3),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded randn on device, N(0,1) bf16; inputs larger than L2, no flush)",
            "config": bench_config(world),
            "prefill": {"ms": round(pre_ms_max, 3), "correction_ms": round(corr_ms, 3),
                        "attention_ms": round(attn_ms_max, 3), "tokens_per_s": round(world * P["L"] * P["B"] /
                                                                                     (pre_ms_max * 1e-3), 1),
                        "attention_tflops": round(attn_tflops, 2),
                        "path": "default: remote scores Q_hi K_hi + Q_hi K_lo + Q_lo K_hi (fp16 hi + lo); query "
                                "block corrected inside the attention kernel, key rows by the correction pass"},
            "decode": {"value": dloop8["gbs_all_ranks"], "unit": "GB/s", "ms": dloop8["ms"],
                       "tokens_per_s": dloop8["tokens_per_s"], "B": Dc["B"],
                       "timing": f"{dloop8['reps']} launches back to back between two CUDA events, mean period",
                       "roofline": {"bound": "hbm", "achieved": dloop8["gbs"],
                                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                    "frac": round(dloop8["gbs"] / peaks["hbm_gbs"], 4),
                                    "traffic": traffic.get("decode", {}).get("bytes_per_launch"),
                                    "peak_source": f"{peak_kind} hbm_gbs"},
                       "clocks": dloop8["clocks"],
                       "batch1": {"ms": dloop1["ms"], "gbs": dloop1["gbs"], "tokens_per_s": dloop1["tokens_per_s"],
                                  "frac": round(dloop1["gbs"] / peaks["hbm_gbs"], 4), "reps": dloop1["reps"],
                                  "clocks": dloop1["clocks"]},
                       "in_step": {"ms": round(dec_ms_max, 4), "gbs": round(dec_gbs_kernel, 1),
                                   "frac": round(dec_gbs_kernel / peaks["hbm_gbs"], 4),
                                   "note": "timed inside the step, right after the prefill kernel"}},
            "prefill_other_paths": paths,
            "prefill_inclusion_exclusion_3pass": ie,
            "plain_rope_same_kernels": {
                "prefill_ms": round(plain_pre_ms, 3),
                "prefill_tflops": round(flop / (plain_pre_ms * 1e-3) / 1e12, 2),
                "decode_ms": round(plain_dec_ms, 4),
                "decode_gbs": round(dbytes / (plain_dec_ms * 1e-3) / 1e9, 1),
            },
            "other_workloads": others,
            "roofline": {"bound": "tensor", "achieved": round(attn_tflops, 2), "peak": tensor_peak,
                         "unit": "TFLOP/s", "frac": round(attn_tflops / tensor_peak, 4),
                         "traffic": traffic.get("prefill_attention", {}).get("bytes_per_launch"),
                         "traffic_smaller_sizes": traffic.get("prefill_attention", {}).get("measured_smaller"),
                         "traffic_note": "DRAM bytes per launch measured by ncu at the profiling sizes (same G and "
                                         "w0 / L); they do not grow in proportion to L, so the 128K launch's "
                                         "traffic is not extrapolated",
                         "kernel": "bifocal_prefill_hilo_kernel<128, false, 0>",
                         "peak_source": f"{peak_kind} bf16_tflops_sustained (kernel timed inside a multi-second loop)",
                         "executed_tflops": round(exec_flop / (attn_ms_max * 1e-3) / 1e12, 2),
                         "executed_frac": round(exec_flop / (attn_ms_max * 1e-3) / 1e12 / tensor_peak, 4),
                         "executed_note": "tensor-core flop actually issued: three score products per remote tile "
                                          "(hi + lo), one per local tile, one P V per tile",
                         "per_ghz": {"kernel_tflops_per_sm_ghz": round(attn_tflops / sm_ghz, 1) if sm_ghz else None,
                                     "kernel_executed_tflops_per_sm_ghz":
                                         round(exec_flop / (attn_ms_max * 1e-3) / 1e12 / sm_ghz, 1) if sm_ghz else None,
                                     "peak_tflops_per_sm_ghz": round(tensor_peak / peak_ghz, 1) if peak_ghz else None,
                                     "tensor_core_tflops_per_sm_ghz": round(8192 * 148 / 1e3, 1),
                                     "note": "TFLOP/s divided by the median SM clock sampled while each ran "
                                             "(the step's clocks for the kernel, the peak file's for cuBLAS); "
                                             "the tensor-core figure is 8192 flop per clock per SM (one "
                                             "128 x 128 x 16 product per 64 clocks, measured) x 148 SMs"}},
            "e2e": e2e,
            "gpu_launches": K * 3,
            "gpu_launches_decode_loops": dloop8["reps"] + dloop1["reps"],
            "clocks": clk,
            "cpu_baseline": cpu,
        }
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return out

# ---------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------

_ORACLE_KV = {}


def _oracle_rows_timed(n_rows, seed=0):
    """Time the fp64 oracle on n_rows query rows (all of one KV head's query
    heads) of the 128K prefill workload; returns (algorithmic flop, seconds).
    The keys and values (one KV head, drawn once) are shared by every call; the
    query rows and their positions come from `seed`."""
    import numpy as np
    import torch
    from oracle import jetlong_oracle as jo
    P = PREFILL
    r = P["Hq"] // P["Hkv"]
    if "kv" not in _ORACLE_KV:
        g0 = torch.Generator("cpu").manual_seed(0)
        kk = torch.randn(P["L"], P["D"], generator=g0).to(torch.bfloat16).double().numpy()
        vv = torch.randn(P["L"], P["D"], generator=g0).to(torch.bfloat16).double().numpy()
        _ORACLE_KV["kv"] = (kk, vv)
    kk, vv = _ORACLE_KV["kv"]
    g = torch.Generator("cpu").manual_seed(seed)
    qq = torch.randn(r, n_rows, P["D"], generator=g).to(torch.bfloat16).double().numpy()
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(P["L"], size=n_rows, replace=False))
    p = jo.BifocalParams(L=P["L"], w0=P["w0"], w_pretrained=P["W"], base=P["base"])
    t = time.perf_counter()
    for h in range(r):
        jo.attention_rows(qq[h], rows, kk, vv, p)
    dt = time.perf_counter() - t
    flop = 4.0 * P["D"] * float(np.sum(rows + 1)) * r
    return flop, dt, rows


def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline_sample(seconds=15.0):
    """The oracle on batches of random query rows (new rows each batch) until
    about `seconds` of CPU time have been spent; TFLOP/s from the algorithmic
    flop of the rows done (each row i costs 4 d (i + 1) flop per head)."""
    _oracle_rows_timed(2, seed=7)  # warm-up (thread pool, first-touch)
    flop_sum, t_sum, rows, batch, seed = 0.0, 0.0, 0, 8, 1
    while t_sum < seconds:
        f, dt, _ = _oracle_rows_timed(batch, seed=seed)
        flop_sum += f
        t_sum += dt
        rows += batch
        seed += 1
        batch = int(max(8, min(256, batch * max(1.0, (seconds - t_sum) / max(dt, 1e-3)) * 0.5)))
    return flop_sum / t_sum / 1e12, rows, t_sum


def cpu_baseline(seconds=15.0):
    """The fp64 oracle, as it stands, on the host cores: a bounded sample of the
    128K prefill workload (all cores, and again on one core), the full prefill
    time extrapolated from it by the causal row-cost sum, and the B 1 decode of
    the 128K decode workload timed in full."""
    import numpy as np
    import torch
    from oracle import jetlong_oracle as jo
    tf, rows, t_sum = cpu_baseline_sample(seconds)
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            tf1, rows1, t1 = cpu_baseline_sample(max(2.0, seconds / 3))
    except ImportError:  # pragma: no cover - threadpoolctl is in the image
        tf1, rows1, t1 = None, 0, 0.0
    full_s = prefill_flop(PREFILL) / (tf * 1e12)
    # decode, B 1, 128K cache, every head and key
    Dc = DECODE
    g = torch.Generator("cpu").manual_seed(3)
    dq = torch.randn(1, Dc["Hq"], Dc["D"], generator=g).to(torch.bfloat16).double().numpy()
    kc = torch.randn(1, Dc["L"], Dc["Hkv"], Dc["D"], generator=g).to(torch.bfloat16).double().numpy()
    vc = torch.randn(1, Dc["L"], Dc["Hkv"], Dc["D"], generator=g).to(torch.bfloat16).double().numpy()
    p = jo.BifocalParams(L=Dc["L"], w0=Dc["w0"], w_pretrained=Dc["W"], base=Dc["base"])
    t = time.perf_counter()
    jo.decode(dq, kc, vc, p)
    dec_s = time.perf_counter() - t
    dbytes = decode_bytes(dict(Dc, B=1))
    return {"value": round(tf, 6), "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
            "sample": f"fp64 oracle, {rows} random query rows x 4 q heads of one KV head of the 128K prefill "
                      f"workload, {t_sum:.1f} s; TFLOP/s from the algorithmic flop of those rows",
            "one_core": None if tf1 is None else {"value": round(tf1, 6), "unit": "TFLOP/s", "cores": 1,
                                                 "sample": f"{rows1} rows, {t1:.1f} s"},
            "prefill_128k_full_s_extrapolated": round(full_s, 1),
            "extrapolation": "full prefill time = its algorithmic flop (sum over rows of 4 d (i + 1) per head) / "
                             "the sampled rate; extrapolated, not run",
            "decode_128k_b1_full": {"s": round(dec_s, 3), "gbs": round(dbytes / dec_s / 1e9, 4),
                                    "tokens_per_s": round(1.0 / dec_s, 4),
                                    "sample": "the whole decode (32 q heads, 131072 keys), timed in full"}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    for _ in range(args.warmup):
        _oracle_rows_timed(2, seed=7)
    times, flops = [], []
    for i in range(args.steps):
        f, dt, _ = _oracle_rows_timed(args.ref_rows, seed=100 + i)
        flops.append(f)
        times.append(dt)
    total = sum(times)
    value = sum(flops) / total / 1e12
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": 1,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded randn, N(0,1) bf16 widened to fp64)",
        "config": bench_config(1),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
                         "sample": f"each step: {args.ref_rows} random query rows x 4 q heads of one KV head of "
                                   f"the 128K prefill workload on the fp64 CPU oracle"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the fp16-single-product and pre-rotated-key prefill measurements")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the 1.7B 64K, tiny and length / band sweep measurements")
    ap.add_argument("--no-ie", action="store_true", help="skip the three-call inclusion-exclusion measurement")
    ap.add_argument("--no-decode-loops", action="store_true",
                    help="report the in-step decode time only (profiling runs: no back-to-back decode loops)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=4)
    ap.add_argument("--prefill-len", type=int, default=None, help="smaller prefill L (profiling runs only)")
    ap.add_argument("--decode-len", type=int, default=None, help="smaller decode L (profiling runs only)")
    ap.add_argument("--decode-batch", type=int, default=None, help="decode batch (default 8)")
    args = ap.parse_args()
    # Smaller profiling sizes keep G = L / w_pretrained and w0 / L of the full workload.
    for cfg, n in ((PREFILL, args.prefill_len), (DECODE, args.decode_len)):
        if n:
            f = n / cfg["L"]
            cfg["W"] = max(1, int(round(cfg["W"] * f)))
            cfg["w0"] = int(round(cfg["w0"] * f))
            cfg["L"] = n
            cfg["workload"] += f" (profiling size L={n}, w_pretrained={cfg['W']}, w0={cfg['w0']})"
    if args.decode_batch:
        DECODE["B"] = args.decode_batch
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        out = run_reference(args)
    else:
        out = run_ours(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
