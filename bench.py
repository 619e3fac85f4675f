"""Benchmark of the MoE-layer forward pass on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle, timed on host cores

A step is one pass of the whole layer (router + softmax + selection ->
dispatch -> grouped expert MLP -> combine) over one batch of synthetic input
through moe_forward, replayed as a CUDA graph; a second timed loop issues
the same layer as the staged C-ABI calls with a CUDA event between stages
for the per-stage split and the grouped MLP's own duration. L2 is flushed
before every timed step, outside the events: a 256 MiB write, then a
256 MiB read so no dirty flush data is left to write back. ``value`` is
tokens/s over the K timed steps (inputs resident in HBM); ``e2e`` repeats
the measurement through moe_forward_host with the activations in pinned
host memory and the copies inside the timed region. Multi-GPU runs are
independent replicas (one process per GPU, no collective on the data path);
the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "ditmoe_xl"
METRIC = "MoE-layer tokens/s and TFLOP/s (or HBM GB/s) vs B200 roofline, 1 GPU"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
# Device-side wait (SM clock cycles, ~0.5-1 ms) enqueued before an eagerly
# issued, event-timed pass, so that the host has enqueued the pass before
# the GPU reaches it.
HOST_AHEAD_CYCLES = 1_000_000


class L2Flush:
    """Leaves L2 cold and clean between timed steps: writes a 256 MiB buffer
    (evicting everything) and then reads another (so the lines left behind
    are clean and the timed step pays no write-back of the flush's own data).
    Runs outside the timed events."""

    def __init__(self, device):
        import torch
        self.a = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.b = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def __call__(self, step=0):
        self.a.fill_(step & 255)
        self.sink = self.b.sum()

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of the grouped-MLP
# launches of one layer pass, from one ncu capture (profiles/), valid only while
# the code of the profiled kernel source and of the headers it shares (comments
# and whitespace aside, see source_hash) is identical to the code captured.
NCU_TRAFFIC = {
    "des_vote": {"bytes": (421.70 + 3.91) * 1e6,
                 "source": "block_sm100.cu", "sha256_16": "e765ef1e3251668c"},
    "ditmoe_xl": {"bytes": (163.55 + 257.40 + 458.85 + 38.43) * 1e6,
                  "source": "gemm_sm100.cu", "sha256_16": "9d171a92bd63626f"},
    "ecdit": {"bytes": (1234.66 + 251.09 + 1472.26 + 58.55) * 1e6,
              "source": "gemm_sm100.cu", "sha256_16": "9d171a92bd63626f"},
    "mmoe": {"bytes": (231.54 + 154.37 + 421.29 + 40.01) * 1e6,
             "source": "gemm_sm100.cu", "sha256_16": "9d171a92bd63626f"},
}


def fused_block(cfg):
    """Whether moe_forward runs this layer as one persistent kernel (the
    library's rule for small blocks: bf16, at most 128 tokens, token choice
    or DES, no shared expert, E <= 128, k <= 32, d <= 32768)."""
    return (cfg["dtype"] == "bf16" and 1 <= cfg["T"] <= 128
            and cfg["routing"] in ("token_topk", "des_vote", "des_seq") and cfg["n_shared"] == 0
            and cfg["E"] <= 128 and cfg["k"] <= 32 and cfg["d"] <= 32768)


def fused_f32(cfg):
    """Whether moe_forward runs this layer as one kernel with a CTA per token
    (the library's rule for small fp32 layers: token choice, no shared
    expert, no mixed constant experts, at most 1024 tokens, k <= 32,
    d <= 1024 and h <= 2048, both multiples of 4)."""
    return (cfg["dtype"] == "f32" and cfg["routing"] == "token_topk" and cfg["n_shared"] == 0
            and not cfg.get("const_mix", 0) and 1 <= cfg["T"] <= 1024 and cfg["E"] <= 128
            and 1 <= cfg["k"] <= min(32, cfg["E"]) and 4 <= cfg["d"] <= 1024 and cfg["d"] % 4 == 0
            and 4 <= cfg["h"] <= 2048 and cfg["h"] % 4 == 0)


# fp32 FMA lanes per SM on B200 (4 SM sub-partitions x 32): the peak of the
# CUDA-core fp32 path is 148 SMs x 128 lanes x 2 FLOP per clock.
FP32_LANES_PER_SM = 128


def forward_launches(cfg):
    """Kernels one moe_forward launches for this workload (the library's
    path choice: one kernel for small fp32 layers and for small bf16 blocks;
    split router + fused routing for other blocks of <= 128 tokens; split
    router for <= 512; else the full router)."""
    if fused_block(cfg) or fused_f32(cfg):
        return 1
    bf16 = cfg["dtype"] == "bf16"
    r = cfg["routing"]
    ec = r == "expert_choice"
    na = (cfg["T"] // cfg["group_size"]) * cfg["E"] * cfg["capacity"] if ec else cfg["T"] * cfg["k"]
    if bf16 and cfg["T"] > 128 and cfg["n_shared"] and cfg["E_heavy"]:
        # shared up projection (side stream), routed up projection, both down projections
        n = 1 + 3
    else:
        n = 1 + StagedLayer._mlp_launches(cfg)  # combine + expert MLP
    if (bf16 and cfg["T"] <= 128 and r in ("token_topk", "des_vote") and cfg["E"] <= 128
            and cfg["k"] <= 32 and cfg["T"] * cfg["k"] <= 2048):
        return n + 2  # split router, then routing + dispatch + gather in one kernel
    if bf16 and cfg["T"] <= 512 and r in ("token_topk", "des_vote"):
        n += 2 + (r == "des_vote")  # split router, finish (+ DES re-route)
    else:
        n += 1 + (r != "token_topk")  # router (+ expert choice / DES vote)
    if ec and (2 * cfg["group_size"] + cfg["E"] * cfg["capacity"]) * 4 <= 48 * 1024:
        n += 1  # closed-form expert-choice dispatch with its token lists, one launch
    else:
        n += (1 if na <= 1024 else 3) + (1 if ec else 0)  # dispatch (+ token lists)
    n += 1 if cfg["E_heavy"] else 0  # row gather
    return n


# Headers every tensor-core kernel source includes (their waits, loads and
# MMAs): a capture is valid only while these are unchanged too.
KERNEL_HEADERS = ("tc_ptx.cuh", "common.cuh")


def code_text(text):
    """C++/CUDA source with comments and whitespace removed: what a capture
    of the compiled kernel depends on (the kernel sources hold no string
    literal with a comment marker in it)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return re.sub(r"\s+", "", text)


def source_hash(name):
    """sha256 prefix of a kernel source together with the headers it shares,
    taken over their code_text (an edit of comments or layout does not
    change what was profiled)."""
    import hashlib
    h = hashlib.sha256()
    for part in (name,) + KERNEL_HEADERS:
        with open(os.path.join(ROOT, "mixture_experts_layer_33_b200", "csrc", part), "rb") as f:
            h.update(code_text(f.read().decode()).encode())
    return h.hexdigest()[:16]


# ------------------------------------------------------------- bookkeeping
def describe(cfg):
    """Workload description for the JSON line."""
    parts = [f"T={cfg['T']}", f"d={cfg['d']}", f"E={cfg['E']}"]
    if cfg["routing"] == "token_topk":
        parts.append(f"top-{cfg['k']}")
    elif cfg["routing"] == "expert_choice":
        parts.append(f"expert-choice S={cfg['group_size']} C={cfg['capacity']}")
    elif cfg["routing"] == "des_seq":
        parts.append(f"DES-Seq K={cfg['k']} k_local={cfg['k_local']}")
    else:
        parts.append(f"DES-Vote K={cfg['k']} M_core={cfg['M_core']}")
    parts.append(f"h={cfg['h']} {cfg['act']}")
    if cfg["n_shared"]:
        parts.append(f"+{cfg['n_shared']} shared h={cfg['h_shared']}")
    if cfg["E_heavy"] != cfg["E"]:
        parts.append(f"{cfg['E'] - cfg['E_heavy']} zero-compute experts")
    return f"{cfg['name']}: " + ", ".join(parts) + f", {cfg['dtype']}"


def mlp_flops(cfg, n_heavy_rows):
    """Algorithmic FLOPs of the grouped MLP: executed heavy rows and shared tokens only."""
    gemm = 6 if cfg["act"] == "swiglu" else 4  # 2*d*h per GEMM; SwiGLU has gate+up+down
    routed = n_heavy_rows * gemm * cfg["d"] * cfg["h"]
    shared = cfg["T"] * 4 * cfg["d"] * cfg["n_shared"] * cfg["h_shared"]
    return routed + shared


def weight_bytes_used(cfg, used_experts):
    """Unique heavy-expert weight bytes one layer pass must read (DES latency model)."""
    per = (3 if cfg["act"] == "swiglu" else 2) * cfg["d"] * cfg["h"] * (2 if cfg["dtype"] == "bf16" else 4)
    return used_experts * per


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def reduce_max_over_ranks(value, dist=None):
    """Max of a float over all ranks (identity without a process group)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank, world, max_seconds):
    return units_per_rank * world / max_seconds


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every few ms by
    NVML from a background thread while the timed region runs; falls back
    to nvidia-smi polling if NVML is unavailable."""

    REASON_BITS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40, "sw_power_cap": 0x4}

    def __init__(self, torch_device, period_s=0.002):
        self.dev = torch_device
        self.period = period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = None
        self._thread = None
        self._smi = None

    def _handle(self, pynvml):
        import torch
        try:
            p = torch.cuda.get_device_properties(self.dev)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.dev.index or 0)

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = self._handle(pynvml)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            self._start_smi()
            return
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    self.samples.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                    bits = int(get_reasons(h))
                    for n, b in self.REASON_BITS.items():
                        if bits & b:
                            self.reasons.add(n)
                except Exception:
                    pass
                time.sleep(self.period)
        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def _start_smi(self):
        self.path = os.path.join("/tmp", f"moe_bench_clocks_{os.getpid()}.csv")
        try:
            self._out = open(self.path, "w")
            self._smi = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=clocks.sm,clocks.max.sm,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self._out, stderr=subprocess.DEVNULL)
        except OSError:
            self._smi = None

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
        elif self._smi is not None:
            self._smi.terminate()
            self._smi.wait(timeout=5)
            self._out.close()
            names = ["hw_slowdown", "sw_thermal_slowdown", "hw_thermal_slowdown", "sw_power_cap"]
            with open(self.path) as f:
                for line in f:
                    cols = [c.strip() for c in line.split(",")]
                    try:
                        self.samples.append(float(cols[0]))
                        self.max_mhz = float(cols[1])
                    except (ValueError, IndexError):
                        continue
                    for n, v in zip(names, cols[2:6]):
                        if v.lower() == "active":
                            self.reasons.add(n)
            os.unlink(self.path)
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ----------------------------------------------------------- GPU benchmark
class StagedLayer:
    """One layer pass as staged C-ABI calls with an event between stages."""

    def __init__(self, m, cfg, inp, device):
        import torch
        self.m, self.cfg, self.inp = m, cfg, inp
        self.c = m.make_config(cfg)
        na = m.num_assignments(self.c)
        T, E, d = cfg["T"], cfg["E"], cfg["d"]
        f = dict(device=device)
        self.logits = torch.empty(T, E, dtype=torch.float32, **f)
        self.probs = torch.empty(T, E, dtype=torch.float32, **f)
        self.sel = torch.empty(na, dtype=torch.int32, **f)
        self.w = torch.empty(na, dtype=torch.float32, **f)
        self.votes = torch.empty(E, dtype=torch.int64, **f)
        self.core = torch.empty(max(1, cfg.get("M_core", 0)), dtype=torch.int32, **f)
        self.core_all = torch.empty(E, dtype=torch.int32, **f)  # DES-Seq: the union, then -1
        self.n_core = torch.empty(1, dtype=torch.int32, **f)
        self.offsets = torch.empty(self.c.n_heavy + 1, dtype=torch.int32, **f)
        self.perm = torch.empty(na, dtype=torch.int32, **f)
        self.row_of = torch.empty(na, dtype=torch.int32, **f)
        ec = cfg["routing"] == "expert_choice"
        self.tok_ptr = torch.empty(T + 1, dtype=torch.int32, **f) if ec else None
        self.tok_assign = torch.empty(na, dtype=torch.int32, **f) if ec else None
        self.x_perm = torch.empty(na, d, dtype=inp["x"].dtype, **f)
        self.y_perm = torch.empty(na, d, dtype=inp["x"].dtype, **f)
        self.y_sh = torch.empty(T, d, dtype=inp["x"].dtype, **f) if cfg["n_shared"] else None
        self.y = torch.empty_like(inp["x"])
        self.ws = m.alloc_workspace(self.c, device)
        self.status = torch.zeros(1, dtype=torch.int32, **f)
        self.stages = ["router+select", "dispatch", "grouped_mlp", "combine"]
        self.launches = {"router+select": 1 + (cfg["routing"] != "token_topk"),
                         "dispatch": (1 if na <= 1024 else 3) + (1 if self.c.n_heavy else 0)
                         + (1 if ec else 0),
                         "grouped_mlp": self._mlp_launches(cfg),
                         "combine": 1}

    @staticmethod
    def _mlp_launches(cfg):
        routed = 1 if cfg["E_heavy"] else 0
        shared = 1 if cfg["n_shared"] else 0
        if cfg["dtype"] != "bf16":
            return 2 * (routed + shared)
        if cfg["T"] <= 128:  # weight-streaming kernel: one launch per problem
            return routed + shared
        if routed and shared:
            return 2 if cfg["act"] == "gelu" else 3
        return 2 * (routed + shared)

    def run_forward(self):
        """The whole layer through the single entry point moe_forward."""
        i = self.inp
        self.m.forward(self.c, i["x"], i["W_r"], i["W1"], i["W2"], self.y, self.ws,
                       residual=i["x"], z_prev=i["z_prev"], bias=i["logit_bias"],
                       Ws1=i["Ws1"], Ws2=i["Ws2"], const_vecs=i["const_vecs"],
                       dev_status=self.status)

    def run(self, events=None):
        m, cfg, i = self.m, self.cfg, self.inp
        r = cfg["routing"]

        def mark(j):
            if events is not None:
                events[j].record()
        mark(0)
        m.router(i["x"], i["W_r"], self.logits, self.probs, bias=i["logit_bias"],
                 z_prev=i["z_prev"], z_prev_scale=cfg["gate_residual_scale"],
                 k=cfg["k"] if r == "token_topk" else 0, renorm=cfg["renorm"],
                 idx=self.sel if r == "token_topk" else None,
                 w=self.w if r == "token_topk" else None)
        if r == "expert_choice":
            m.select_expert_choice(self.probs, cfg["group_size"], cfg["capacity"], self.sel, self.w)
        elif r == "des_vote":
            m.core_set_vote(self.probs, cfg["k"], cfg["M_core"], self.votes, self.core, self.sel, self.w)
        elif r == "des_seq":
            m.core_set_union(self.probs, cfg["k"], cfg["k_local"], self.core_all, self.n_core,
                             self.sel, self.w)
        mark(1)
        m.dispatch(self.c, self.sel, i["x"], self.x_perm, self.offsets, self.perm, self.row_of,
                   self.tok_ptr, self.tok_assign, self.status, self.ws)
        mark(2)
        m.grouped_mlp(self.c, self.x_perm, self.offsets, i["W1"], i["W2"], i["x"], i["Ws1"],
                      i["Ws2"], self.y_perm, self.y_sh, self.status, self.ws)
        mark(3)
        m.combine(self.c, self.y_perm, self.y_sh, self.sel, self.w, self.row_of, self.tok_ptr,
                  self.tok_assign, i["x"], i["const_vecs"], i["x"], self.y, self.status)
        mark(4)


# The other workloads measured beside the headline one, each timed exactly
# like it (the CPU oracle is timed for the headline workload only).
SECONDARY_WORKLOADS = ("ecdit", "des_vote", "mmoe", "mmoe_skewed", "tiny_fp32")


def measure_workload(m, gen, name, dev, args, world, dist, rank):
    """One workload: the layer as a CUDA graph (value), the staged calls
    (stage split and the dominant kernel's roofline), the fused one-launch
    layers eagerly, and the host-buffer path (e2e). Returns the fields of
    its JSON line and the host inputs (for the CPU oracle)."""
    import torch

    cfg = gen.workload(name)
    inp = gen.make_inputs(cfg, dev)
    layer = StagedLayer(m, cfg, inp, dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        flush(1)
        layer.run()
    torch.cuda.synchronize()
    if int(layer.status.item()) != 0:
        raise RuntimeError(f"device status {int(layer.status.item())} ({name})")

    # Executed heavy rows and used experts (fixed by the seeded inputs).
    offs = layer.offsets.cpu().tolist()
    n_rows = offs[-1]
    used = sum(1 for a, b in zip(offs[:-1], offs[1:]) if b > a)
    flops = mlp_flops(cfg, n_rows)

    # The layer (moe_forward) as one CUDA graph; eager if capture is refused.
    for _ in range(2):
        layer.run_forward()
    torch.cuda.synchronize()
    graph = None
    if not args.no_graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                layer.run_forward()
            for _ in range(3):
                flush(1)
                graph.replay()
            torch.cuda.synchronize()
        except Exception as exc:  # noqa: BLE001
            graph = None
            print(f"graph capture unavailable: {exc}", file=sys.stderr)

    # Timed region 1 (value): K layer passes, L2 flushed before each.
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    sampler = ClockSampler(dev)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for s in range(args.steps):
        flush(s)
        ev[s][0].record()
        if graph is not None:
            graph.replay()
        else:
            layer.run_forward()
        ev[s][1].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = sum(a.elapsed_time(b) for a, b in ev)
    max_s = reduce_max_over_ranks(total_ms / 1e3, dist if world > 1 else None)
    ms_per_step = max_s * 1e3 / args.steps
    value = aggregate_throughput(cfg["T"] * args.steps, world, max_s)
    graphed = graph is not None
    del graph

    # Timed region 2: the same passes as staged calls with an event between
    # stages, for the per-stage split and the dominant kernel's duration. The
    # stages are enqueued one host call at a time (tensor-map encoding and
    # launch set-up on the host), so a short device-side wait after the L2
    # flush lets the host enqueue the whole pass first: the events then time
    # the GPU work of each stage, not the GPU waiting for the host.
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    for s in range(args.steps):
        flush(s)
        torch.cuda._sleep(HOST_AHEAD_CYCLES)
        layer.run(sev[s])
    torch.cuda.synchronize()
    stage_ms = {n: 0.0 for n in layer.stages}
    for s in range(args.steps):
        for j, n in enumerate(layer.stages):
            stage_ms[n] += sev[s][j].elapsed_time(sev[s][j + 1])

    # Timed region 3 (small fused blocks): moe_forward issued eagerly with
    # events around it; its one kernel (after a memset of its sync words) is
    # the dominant launch, so this bounds that kernel's duration from above.
    fused_ms = None
    if fused_block(cfg) or fused_f32(cfg):
        fev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        torch.cuda.synchronize()
        for s in range(args.steps):
            flush(s)
            torch.cuda._sleep(HOST_AHEAD_CYCLES)
            fev[s][0].record()
            layer.run_forward()
            fev[s][1].record()
        torch.cuda.synchronize()
        fused_ms = sum(a.elapsed_time(b) for a, b in fev) / args.steps

    # End to end through moe_forward_host: pinned host activations, copies timed.
    x_h = inp["x"].cpu().pin_memory()
    zp_h = inp["z_prev"].cpu().pin_memory() if inp["z_prev"] is not None else None
    y_h = torch.empty_like(x_h).pin_memory()
    ws = m.alloc_workspace(layer.c, dev)

    def e2e_step():
        m.forward_host(layer.c, x_h, inp["W_r"], inp["W1"], inp["W2"], y_h, ws,
                       residual_host=x_h, z_prev_host=zp_h, bias=inp["logit_bias"],
                       Ws1=inp["Ws1"], Ws2=inp["Ws2"], const_vecs=inp["const_vecs"],
                       dev_status=layer.status)
    for _ in range(max(3, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    e2e_ms = 0.0
    for s in range(args.steps):
        flush(s)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b.record(stream)
        b.synchronize()
        e2e_ms += a.elapsed_time(b)
    e2e_s = reduce_max_over_ranks(e2e_ms / 1e3, dist if world > 1 else None)
    act_bytes = cfg["T"] * cfg["d"] * inp["x"].element_size()
    h2d = act_bytes + (cfg["T"] * cfg["E"] * 4 if zp_h is not None else 0)
    if int(layer.status.item()) != 0:
        raise RuntimeError(f"device status {int(layer.status.item())} ({name})")

    peaks, peak_src = load_peaks()
    tr = NCU_TRAFFIC.get(cfg["name"])
    traffic = tr["bytes"] if tr and tr["sha256_16"] == source_hash(tr["source"]) else None
    gm_ms = stage_ms["grouped_mlp"] / args.steps  # grouped-MLP launches, from timed region 2
    if fused_f32(cfg) and fused_ms is not None:
        # One kernel on CUDA cores: fp32 FMAs against the fp32 lanes' peak at
        # the maximum SM clock (latency-bound at these sizes).
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        pk = sms * FP32_LANES_PER_SM * 2 * (clocks.get("sm_max_mhz") or 1965.0) * 1e6 / 1e12
        achieved = flops / (fused_ms / 1e3) / 1e12
        roof = {"bound": "alu", "kernel": "small_f32_kernel (whole layer, one launch after a memset)",
                "achieved": round(achieved, 2), "peak": round(pk, 1), "unit": "TFLOP/s",
                "frac": round(achieved / pk, 4), "traffic": None, "algorithmic_per_launch": flops,
                "peak_source": f"derived: {sms} SMs x {FP32_LANES_PER_SM} fp32 lanes x 2 FLOP x max SM clock"}
    elif cfg["dtype"] == "bf16" and cfg["T"] <= 128:  # small blocks stream expert weights
        bytes_ = weight_bytes_used(cfg, used)
        if fused_ms is not None:
            kname = "moe_block_kernel (whole layer, one launch after a memset)"
            achieved = bytes_ / (fused_ms / 1e3) / 1e9
        else:
            kname = "expert_stream_kernel (weight-streaming expert MLP, one launch)"
            achieved = bytes_ / (gm_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": kname,
                "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                "algorithmic_per_launch": bytes_, "peak_source": peak_src}
    else:
        achieved = flops / (gm_ms / 1e3) / 1e12
        pk = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "kernel": "grouped_mlp (GEMM1 + GEMM2 launches)",
                "achieved": round(achieved, 1), "peak": pk, "unit": "TFLOP/s",
                "frac": round(achieved / pk, 4), "traffic": traffic,
                "algorithmic_per_launch": flops, "peak_source": peak_src + " (burst)"}

    out = {
        "value": round(value, 1), "unit": "tokens/s", "ms_per_step": round(ms_per_step, 4),
        "dtype": cfg["dtype"], "config": bench_config(cfg, world),
        "layer_tflops": round(flops / (ms_per_step / 1e3) / 1e12, 1),
        "layer_weight_gbs": round(weight_bytes_used(cfg, used) / (ms_per_step / 1e3) / 1e9, 1),
        "cuda_graph": graphed,
        "stage_ms": {k: round(v / args.steps, 4) for k, v in stage_ms.items()},
        "fused_layer_ms": round(fused_ms, 4) if fused_ms is not None else None,
        "heavy_rows": n_rows, "experts_used": used,
        "roofline": roof,
        "e2e": {"value": round(aggregate_throughput(cfg["T"] * args.steps, world, e2e_s), 1),
                "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": act_bytes,
                "api": "moe_forward_host"},
        "gpu_launches": forward_launches(cfg) * args.steps,
        "clocks": clocks,
    }
    hin = {k: gen.to_numpy_f32(v) for k, v in inp.items()} if rank == 0 else None
    del layer, inp, ws, flush
    torch.cuda.empty_cache()
    return cfg, out, hin


def bench_config(cfg, world):
    """The ``config`` object of a JSON line (the same for both arms)."""
    return {"workload": describe(cfg), "global_batch_tokens": cfg["T"] * world,
            "parallelism": "replicas" if world > 1 else "single GPU",
            "l2": "flushed before every timed step (256 MiB write, then 256 MiB read so L2 is left clean)"}


def gpu_bench(args):
    import torch
    import torch.distributed as dist

    from mixture_experts_layer_33_b200 import inputs as gen
    from mixture_experts_layer_33_b200 import moe as m

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if m.device_check(local) != m.MOE_OK:
        raise RuntimeError("not an sm_100 GPU")

    cfg, res, hin = measure_workload(m, gen, args.workload, dev, args, world, dist, rank)
    line = {"metric": METRIC, "value": res["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": res["dtype"], "data": "synthetic (seeded Gaussian inputs, random-init weights)"}
    line.update({k: v for k, v in res.items() if k not in line})
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, hin, budget_s=args.cpu_budget)
    hin = None
    if args.workload == DEFAULT_WORKLOAD and not args.headline_only:
        # The other workloads, each timed like the headline one; the total
        # launches of the run include theirs.
        line["workloads"] = {}
        for name in SECONDARY_WORKLOADS:
            _, r2, _ = measure_workload(m, gen, name, dev, args, world, dist, rank=1)
            line["workloads"][name] = r2
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------- oracle (CPU) timing
def _oracle_sample(cfg, hin, n_tokens):
    """The oracle's full layer (its own fp64 routing) on the first tokens.

    Token choice: per-token routing, so any prefix is exact. Expert choice:
    whole routing groups. DES: the whole block.
    """
    import oracle
    if cfg["routing"] == "expert_choice":
        S = cfg["group_size"]
        n_tokens = max(S, (n_tokens // S) * S)
    if cfg["routing"] == "des_vote":
        n_tokens = cfg["T"]
    n = min(n_tokens, cfg["T"])
    sub = dict(cfg, T=n)
    zp = hin["z_prev"][:n] if hin["z_prev"] is not None else None
    sel = oracle.route(sub, hin["x"][:n], hin["W_r"], hin["logit_bias"], zp)
    y = oracle.forward(sub, hin["x"][:n], hin["W1"], hin["W2"], sel, cfg["kinds"],
                       hin["const_vecs"], hin["Ws1"], hin["Ws2"], residual=hin["x"][:n])
    return n, y


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def cpu_baseline(cfg, hin, budget_s=15.0):
    """Time the oracle as it stands on a bounded sample (grows until ~budget_s)."""
    n = 64 if cfg["routing"] == "token_topk" else 1
    best = None
    t_total = 0.0
    while True:
        t0 = time.perf_counter()
        done, _ = _oracle_sample(cfg, hin, n)
        dt = time.perf_counter() - t0
        t_total += dt
        best = (done, dt)
        if done >= cfg["T"] or dt >= budget_s / 3 or t_total >= budget_s:
            break
        n *= 2
    done, dt = best
    return {"value": round(done / dt, 2), "unit": "tokens/s", "cores": _cores(), "kind": "oracle",
            "sample": f"fp64 numpy oracle, own routing, first {done} of {cfg['T']} tokens "
                      f"({dt:.1f} s)"}


def reference_bench(args):
    """--impl reference: the oracle on the host cores, same metric/config."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch

    from mixture_experts_layer_33_b200 import inputs as gen
    cfg = gen.workload(args.workload)
    hin = {k: gen.to_numpy_f32(v) for k, v in gen.make_inputs(cfg, "cpu").items()}
    # Per-step sample sized so K + W steps finish in a few minutes.
    n = 64 if cfg["routing"] == "token_topk" else 1
    t0 = time.perf_counter()
    done, _ = _oracle_sample(cfg, hin, n)
    probe = time.perf_counter() - t0
    per_step_budget = max(1.0, 120.0 / max(1, args.steps + args.warmup))
    if cfg["routing"] == "token_topk" and probe < per_step_budget:
        n = int(n * min(64, per_step_budget / max(probe, 1e-3)))
    for _ in range(args.warmup):
        _oracle_sample(cfg, hin, n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        done, _ = _oracle_sample(cfg, hin, n)
    dt = time.perf_counter() - t0
    v = done * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3 / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(cfg, world),
        "cpu_baseline": {"value": round(v, 2), "unit": "tokens/s", "cores": _cores(),
                         "kind": "oracle",
                         "sample": (f"fp64 numpy oracle, own routing, first {done} of {cfg['T']} "
                                    "tokens per step (a token's output depends only on its own "
                                    "routing under token choice, so any prefix is exact)"
                                    if cfg["routing"] == "token_topk" else
                                    f"fp64 numpy oracle, own routing, first {done} of {cfg['T']} "
                                    "tokens per step (whole routing groups / blocks)")},
        "e2e": {"value": round(v, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "torch_threads": torch.get_num_threads(),
    }
    print(json.dumps(line), flush=True)


def des_sweep(args):
    """DES page, sections 3.3 and 4.2: the small block under vanilla top-8,
    DES-Seq and DES-Vote, for blocks of N = 8..64 tokens on the skewed
    synthetic logits. Per N and routing: U (experts that get rows, so
    weights read), the layer time (moe_forward as a CUDA graph, L2
    flushed clean before every step) and U * 12.58 MB / time. One JSON line;
    not part of the driver's contract."""
    import torch

    from mixture_experts_layer_33_b200 import inputs as gen
    from mixture_experts_layer_33_b200 import moe as m

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    variants = [("vanilla top-8", "des_vanilla", {}),
                ("DES-Seq k_local=1", "des_seq", {"k_local": 1}),
                ("DES-Seq k_local=2", "des_seq", {"k_local": 2}),
                ("DES-Vote beta=0.5", "des_vote", {})]
    rows = []
    for N in (8, 16, 32, 64):
        for label, name, over in variants:
            cfg = gen.workload(name, T=N, **over)
            inp = gen.make_inputs(cfg, dev)
            c = m.make_config(cfg)
            ws = m.alloc_workspace(c, dev)
            y = torch.empty_like(inp["x"])
            status = torch.zeros(1, dtype=torch.int32, device=dev)
            offsets = torch.empty(c.n_heavy + 1, dtype=torch.int32, device=dev)

            def fwd(aux=None):
                m.forward(c, inp["x"], inp["W_r"], inp["W1"], inp["W2"], y, ws,
                          residual=inp["x"], bias=inp["logit_bias"], aux=aux,
                          dev_status=status)
            fwd({"offsets": offsets})
            torch.cuda.synchronize()
            offs = offsets.cpu().tolist()
            U = sum(1 for a, b in zip(offs[:-1], offs[1:]) if b > a)
            for _ in range(args.warmup):
                fwd()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fwd()
            times = []
            for s in range(args.steps):
                flush(s)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                g.replay()
                b.record()
                b.synchronize()
                times.append(a.elapsed_time(b) * 1e3)
            del g
            if int(status.item()) != 0:
                raise RuntimeError(f"device status {int(status.item())} for {label} N={N}")
            us = statistics.median(times)
            wbytes = U * 3 * cfg["d"] * cfg["h"] * 2
            rows.append({"N": N, "routing": label, "U": U, "layer_us": round(us, 1),
                         "weight_gbs": round(wbytes / (us / 1e6) / 1e9, 1)})
    for N in (8, 16, 32, 64):
        van = next(r for r in rows if r["N"] == N and r["routing"].startswith("vanilla"))
        for r in rows:
            if r["N"] == N:
                r["latency_vs_vanilla"] = round(r["layer_us"] / van["layer_us"], 3)
    print(json.dumps({"sweep": "DES block: vanilla vs DES-Seq vs DES-Vote",
                      "workload": describe(gen.workload("des_vote")), "steps": args.steps,
                      "l2": "flushed clean before every step", "rows": rows}), flush=True)


def ec_sweep(args):
    """EC-DiT page, "Expert-Choice routing" and "capacity factor": the
    expert-choice layer (T=8192, d=2048, E=32, h=8192) with the routing
    group per sequence (S=128) or the whole batch (S=8192) and capacity
    factors f_c in {1, 2, 4} (C = f_c*S/E). Per variant: layer time, grouped
    MLP TFLOP/s and the histogram of experts per token (a token may get 0
    or several experts under expert choice). One JSON line; not part of the
    driver's contract."""
    import torch

    from mixture_experts_layer_33_b200 import inputs as gen
    from mixture_experts_layer_33_b200 import moe as m

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    rows = []
    for S in (128, 8192):
        for fc in (1, 2, 4):
            C = fc * S // 32
            cfg = gen.workload("ecdit", group_size=S, capacity=C)
            inp = gen.make_inputs(cfg, dev)
            c = m.make_config(cfg)
            na = m.num_assignments(c)
            ws = m.alloc_workspace(c, dev)
            y = torch.empty_like(inp["x"])
            status = torch.zeros(1, dtype=torch.int32, device=dev)
            sel = torch.empty(na, dtype=torch.int32, device=dev)

            def fwd(aux=None):
                m.forward(c, inp["x"], inp["W_r"], inp["W1"], inp["W2"], y, ws,
                          residual=inp["x"], aux=aux, dev_status=status)
            fwd({"sel": sel})
            torch.cuda.synchronize()
            per_token = torch.bincount(sel.long(), minlength=cfg["T"]).cpu()
            hist = torch.bincount(per_token).tolist()
            for _ in range(args.warmup):
                fwd()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fwd()
            times = []
            for s_ in range(args.steps):
                flush(s_)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                g.replay()
                b.record()
                b.synchronize()
                times.append(a.elapsed_time(b))
            del g, ws
            if int(status.item()) != 0:
                raise RuntimeError(f"device status {int(status.item())} for S={S} f_c={fc}")
            ms = statistics.median(times)
            flops = mlp_flops(cfg, na)
            rows.append({"S": S, "f_c": fc, "C": C, "assignments": na, "layer_ms": round(ms, 4),
                         "tokens_per_s": round(cfg["T"] / (ms / 1e3), 1),
                         "layer_tflops": round(flops / (ms / 1e3) / 1e12, 1),
                         "experts_per_token_hist": hist})
            torch.cuda.empty_cache()
    print(json.dumps({"sweep": "EC-DiT expert choice: routing group x capacity factor",
                      "workload": describe(gen.workload("ecdit")), "steps": args.steps,
                      "l2": "flushed clean before every step", "rows": rows}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches, not a CUDA graph")
    ap.add_argument("--headline-only", action="store_true",
                    help="measure the named workload only (no 'workloads' entries)")
    ap.add_argument("--des-sweep", action="store_true",
                    help="vanilla vs DES-Seq vs DES-Vote over block sizes (one JSON line)")
    ap.add_argument("--ec-sweep", action="store_true",
                    help="expert choice: routing group x capacity factor (one JSON line)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.des_sweep:
        des_sweep(args)
    elif args.ec_sweep:
        ec_sweep(args)
    elif args.impl == "reference":
        reference_bench(args)
    else:
        gpu_bench(args)


if __name__ == "__main__":
    main()
