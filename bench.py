#!/usr/bin/env python
"""Benchmark of the ternary routed-expert MoE hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl bitmoe|reference]

A step is one pass of the whole hot path -- int8 activation quantization,
router top-k, fused gate+up mat-vec with SwiGLU/requant, down mat-vec with
the top-k combine -- for one batch of tokens through one MoE layer.  Steps
rotate through a stack of layers (and a pool of inputs) whose bytes touched
per rotation exceed twice the L2 size, so every step reads its weights from
HBM, as a decode through consecutive layers does.  The K timed steps are
replayed from CUDA graphs; one JSON line is printed by rank 0.

With N > 1 (torchrun), every rank runs an independent replica on its own GPU
(weak scaling, no collective on the data path); the timed region is bracketed
by barriers and the max over ranks is reported.

--impl reference times the CPU oracle (single-threaded C) on the host, each
step being a bounded sample of the same workload (see `run_reference`).
"""
import argparse
import hashlib
import json
import math
import os
import re
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed-expert decode tok/s per MoE layer; achieved HBM GB/s vs 8 TB/s"
L2_BYTES = 126 * 2 ** 20
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="large",
                    help="tiny | 30b | 30b-b16 | large | large-b8 | 30b-prefill | 30b-sign | large-sign-b8 | "
                         "30b-e16 | large-e16-b8")
    ap.add_argument("--impl", default="bitmoe", choices=["bitmoe", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-suite", action="store_true",
                    help="time only --workload (by default the large-layer run also times the large layer "
                         "at 8 tokens, the 30B-class layer at 1 and 16 tokens and its 2048-token prefill)")
    ap.add_argument("--layers", type=int, default=0,
                    help="layers in the rotated stack (default: enough to exceed 2x L2)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# --------------------------------------------------------------------------- bytes
def kernel_bytes(wl, unique_experts):
    """Algorithmic bytes per launch of each kernel for one step (each byte
    counted once: weights of the unique routed experts, activations in, results
    out)."""
    T, H, F, E, K = wl.ntok, wl.hidden, wl.ffn, wl.n_experts, wl.top_k
    pairs = T * K
    weights = unique_experts * wl.expert_bytes
    kb = {
        # the whole one-token step in one kernel: router, x, the routed
        # experts' packed weights, the int8 intermediates and y
        "step1": E * H * 4 + T * H * 4 + weights + 2 * (pairs * F + pairs * F // 32 * 4)
        + T * H + T * H // 32 * 4 + T * E * 4 + pairs * 8 + T * H * 4,
        "prefill_gateup": unique_experts * 2 * wl.matrix_bytes(F, H) + T * H + T * H // 32 * 4
        + pairs * F + pairs * F // 32 * 4,
        "prefill_down": unique_experts * wl.matrix_bytes(H, F) + pairs * F + pairs * F // 32 * 4 + pairs * H * 4,
        "prefill_gather": pairs * H + pairs * H // 32 * 4,
        "combine": pairs * H * 4 + T * H * 4 + pairs * 4,
        "route": E * H * 4 + T * H * 4 + T * H + T * H // 32 * 4 + T * E * 4 + pairs * 8,
        "quant_act_q8": T * H * 4 + T * H + T * H // 32 * 4,
        "router_logits": E * H * 4 + T * H * 4 + T * E * 4,
        "topk_softmax": T * E * 4 + pairs * 8,
        "router_quant": E * H * 4 + T * H * 4 + T * E * 4 + T * H + T * H // 32 * 4,
        "topk_group": T * E * 4 + pairs * 8 + pairs * 4 * 3,
        "route_group": E * H * 4 + T * H * 4 + 2 * T * E * 4 + T * H + T * H // 32 * 4 + pairs * 8 + pairs * 4 * 3,
        "group": pairs * 4 * 3,
        "gateup": unique_experts * 2 * wl.matrix_bytes(F, H) + T * H + T * H // 32 * 4
        + pairs * F + pairs * F // 32 * 4 + pairs * 8,
        "down": unique_experts * wl.matrix_bytes(H, F) + pairs * F + pairs * F // 32 * 4
        + pairs * H * 4 * 2 + T * H * 4 + pairs * 8,
    }
    # the tensor-core mat-vecs move the same bytes as the CUDA-core ones
    kb["tc_gateup"], kb["tc_down"] = kb["gateup"], kb["down"]
    if wl.shared_ffn:
        # the shared expert's two kernels (gate/up with the requantization,
        # down with the add into y), per launch on average: 8-bit codes plus
        # an fp16 scale per 32 weights, activations in and out
        Fs = wl.shared_ffn
        kb["shared"] = (3 * H * Fs * 34 // 32 + T * H * 5 // 4 + T * Fs * 5 // 2 + T * H * 8) / 2
        # one token: the one-token step reads the shared expert's weights too
        # (and publishes its blocks as tagged words)
        kb["step1"] += 3 * H * Fs * 34 // 32 + Fs // 32 * 10 * 8 * 2
    return kb


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every `period` s
    on a background thread (started before, stopped after the timed region)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_dev, period=0.002):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_dev).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report what is known
            self.err = repr(e)
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()
        return False

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "note": getattr(self, "err", "no samples")}
        s = sorted(self.samples)
        return {"sm_mhz": s[len(s) // 2], "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(s)}


# --------------------------------------------------------------------------- traffic
_CODE_TOKENS = re.compile(r'"(?:\\.|[^"\\\n])*"|//[^\n]*|/\*.*?\*/', re.S)


# The translation unit that defines each kernel of the kernel_bytes table.
KERNEL_SOURCE = {
    "step1": "step1.cu", "gateup": "decode.cu", "down": "decode.cu", "route_group": "decode.cu",
    "topk_group": "decode.cu", "group": "decode.cu", "router_quant": "router.cu", "router_logits": "router.cu",
    "topk_softmax": "router.cu", "prefill_gateup": "prefill.cu", "prefill_down": "prefill.cu",
    "prefill_gather": "prefill.cu", "combine": "prefill.cu", "quant_act_q8": "quant.cu",
    "shared_gateup": "shared.cu", "shared_down": "shared.cu", "shared": "shared.cu", "tc_gateup": "tcmv.cu",
    "tc_down": "tcmv.cu", "route": "decode2.cu"}
_INCLUDE = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)


def _source_closure(name, csrc):
    """name and the local headers it includes, transitively."""
    seen, todo = set(), [name]
    while todo:
        n = todo.pop()
        path = os.path.join(csrc, n)
        if n in seen or not os.path.exists(path):
            continue
        seen.add(n)
        with open(path, encoding="utf-8") as f:
            todo.extend(_INCLUDE.findall(f.read()))
    return sorted(seen)


def kernel_source_hash(kernel=None):
    """Hash of the code of the translation unit that defines `kernel` (and the
    headers it includes), or of every kernel source without a kernel: comments
    dropped and runs of white space collapsed, so that counters taken on a
    kernel stay attributed to it while neither its code nor that of the
    headers it includes changes."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_moe_b200", "csrc")
    tu = KERNEL_SOURCE.get(kernel) if kernel else None
    names = _source_closure(tu, csrc) if tu else sorted(os.listdir(csrc))
    for name in names:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        code = _CODE_TOKENS.sub(lambda m: m.group(0) if m.group(0).startswith('"') else " ", text)
        h.update(name.encode() + b"\0" + " ".join(code.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, if it was taken on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[kernel][workload]
        if e.get("source_hash") != kernel_source_hash(kernel):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


def ncu_field(kernel, workload, field):
    """Another figure of the committed ncu summary (e.g. the tensor-pipe
    utilisation), under the same source-hash rule as ncu_traffic."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[kernel][workload]
        if e.get("source_hash") != kernel_source_hash(kernel):
            return None
        return float(e[field])
    except Exception:
        return None


# --------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The CPU oracle on the host cores, timed as the step of this workload.

    Each step is a bounded sample of one step of the workload: the oracle's
    activation quantization and router for one token plus the expert FFN of
    one of that token's top-k slots (a 1/top_k share of the token's expert
    work), so K steps stay within minutes.  The rate is reported in tokens/s
    by counting each step as 1/top_k token."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import numpy as np
    import oracle
    import synthetic
    wl = synthetic.WORKLOADS[args.workload]
    H, F, K = wl.hidden, wl.ffn, wl.top_k
    wr = synthetic.router(wl, 0).numpy()
    n_tok = 8
    x = synthetic.activations(wl, 0, ntok=n_tok).numpy()
    idx, wts = oracle.route_topk(x, wr, K)
    experts = sorted(set(int(e) for e in idx.ravel()))
    remap = {e: i for i, e in enumerate(experts)}
    wg = np.concatenate([synthetic.expert_matrix(wl, 0, "gate", e).numpy() for e in experts])
    wu = np.concatenate([synthetic.expert_matrix(wl, 0, "up", e).numpy() for e in experts])
    wd = np.concatenate([synthetic.expert_matrix(wl, 0, "down", e).numpy() for e in experts])
    layer = oracle.Layer.from_float(H, F, len(experts), 1, wg, wu, wd, fmt=wl.fmt)

    def step(j):
        t, slot = (j // K) % n_tok, j % K
        xt = x[t:t + 1]
        xq, xd = oracle.quant_act_q8(xt)
        i2, w2 = oracle.route_topk(xt, wr, K)
        e = remap[int(i2[0, slot])]
        oracle.expert_ffn(layer, xq, xd, np.array([[e]], np.int32),
                          w2[:, slot:slot + 1].astype(np.float32))

    with PinnedToOneCore() as pin:
        for j in range(args.warmup):
            step(j)
        t0 = time.perf_counter()
        for j in range(args.steps):
            step(args.warmup + j)
        dt = time.perf_counter() - t0
    value = args.steps / K / dt
    sample = ("each step: oracle act quant + router for 1 token of %s and the expert FFN of one of "
              "its %d slots (counted as 1/%d token), single-threaded, pinned to one core"
              % (wl.describe(), K, K))
    nproc, model = host_cpu()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(wl, None),
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": 1, "kind": "oracle",
                         "sample": sample, "pinned_core": pin.core, "nproc": nproc, "cpu_model": model},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- our arm
def max_over_ranks(ms, world, device=None):
    """The slowest rank's time (ms): the job is done when every replica is."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(tokens_per_rank, world, ms):
    """Whole-job throughput: the tokens every rank processed over the slowest
    rank's time."""
    return world * tokens_per_rank / (ms / 1e3)


def workload_config(wl, layers):
    c = {"workload": wl.describe(), "hidden": wl.hidden, "expert_ffn": wl.ffn,
         "experts": wl.n_experts, "top_k": wl.top_k, "tokens_per_step": wl.ntok,
         "weights": {"sign": "1-bit sign codes, 256-blocks (32 B of signs + fp16 absmean scale), N(0,%g)",
                     "e16": "ternary digits with two-level scales (fp16 anchor per row, 4-bit sub-scale "
                            "per 16 weights), N(0,%g)"}.get(
                         wl.fmt, "ternary absmean 256-blocks (52 B base-3 + fp16 scale), N(0,%g)") % wl.w_std,
         "activations": "x ~ N(0,1) fp32, int8 32-blocks"}
    if layers is not None:
        c["layer_stack"] = layers
        c["l2"] = "inputs larger than L2: %d-layer stack rotated per step" % layers
    return c


def stack_size(wl, step_bytes):
    need = int(math.ceil(2 * L2_BYTES / max(step_bytes, 1)))
    return max(wl.layers, min(need, 64))


def host_cpu():
    """(nproc, CPU model) of this host."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count() or 1, model


class PinnedToOneCore:
    """Pins this process to one core for the duration of a CPU measurement
    (what `taskset -c <core>` does for a child), then restores the affinity."""

    def __enter__(self):
        self.saved = None
        self.core = None
        try:
            self.saved = os.sched_getaffinity(0)
            self.core = max(self.saved)
            os.sched_setaffinity(0, {self.core})
        except (AttributeError, OSError):
            pass
        return self

    def __exit__(self, *a):
        if self.saved is not None:
            try:
                os.sched_setaffinity(0, self.saved)
            except OSError:
                pass
        return False


def cpu_baseline(wl, repeats=3, n_tok=None):
    """The oracle as it stands, single-threaded and pinned to one core, on a
    bounded sample of this workload: the first `n_tok` tokens of the
    workload's inputs in decode batches of the workload's size (8-token
    chunks for prefill).  The routed experts' weights are packed once,
    untimed; the sample is then timed `repeats` times and the median taken."""
    import numpy as np
    import oracle
    import synthetic
    H, F, K = wl.hidden, wl.ffn, wl.top_k
    chunk = wl.ntok if wl.ntok <= 64 else 8
    if n_tok is None:
        big = wl.hidden * wl.ffn >= 4096 * 2048
        n_tok = chunk * (1 if chunk >= 8 else (2 if big else 4))
    wr = synthetic.router(wl, 0).numpy()
    x = synthetic.activations(wl, 0, ntok=max(n_tok, 1)).numpy()[:n_tok]
    idx, _ = oracle.route_topk(x, wr, K)
    e_used = sorted(set(int(e) for e in idx.ravel()))
    layer = oracle.Layer.from_float(
        H, F, len(e_used), K,
        np.concatenate([synthetic.expert_matrix(wl, 0, "gate", e).numpy() for e in e_used]),
        np.concatenate([synthetic.expert_matrix(wl, 0, "up", e).numpy() for e in e_used]),
        np.concatenate([synthetic.expert_matrix(wl, 0, "down", e).numpy() for e in e_used]),
        fmt=wl.fmt)
    remap = np.full(wl.n_experts, -1, np.int32)
    remap[e_used] = np.arange(len(e_used))

    def sample():
        t0 = time.perf_counter()
        for n in range(0, n_tok, chunk):
            toks = x[n:n + chunk]
            xq, xd = oracle.quant_act_q8(toks)
            i2, w2 = oracle.route_topk(toks, wr, K)
            oracle.expert_ffn(layer, xq, xd, remap[i2], w2.astype(np.float32))
        return time.perf_counter() - t0

    with PinnedToOneCore() as pin:
        times = [sample() for _ in range(repeats)]
    med = sorted(times)[len(times) // 2]
    nproc, model = host_cpu()
    return {"value": n_tok / med, "unit": "tok/s", "cores": 1, "kind": "oracle",
            "sample": "%d tokens in batches of %d of %s (layer 0), oracle single-threaded, pinned to one "
                      "core, median of %d timings; weight packing untimed" % (n_tok, chunk, wl.describe(), repeats),
            "times_s": times, "pinned_core": pin.core, "nproc": nproc, "cpu_model": model}


# --------------------------------------------------------------------------- one workload
def routing_histogram(B, x, router, wl):
    """Per-expert count of (token, slot) pairs of one step's routing."""
    import torch
    idx, _ = B.moe_route_topk(x, router, wl.top_k)
    counts = torch.bincount(idx.flatten().long(), minlength=wl.n_experts).cpu().tolist()
    used = [c for c in counts if c]
    return {"counts": counts, "unique_experts": len(used), "max_pairs": max(used),
            "mean_pairs_per_used_expert": sum(used) / len(used)}


def build_stack(B, wl, n_layers, dev, seed_off):
    from bit_moe_b200.layers import quantize_layer
    import synthetic
    layers, routers = [], []
    for l in range(n_layers):
        fn = lambda role, e, l=l: synthetic.expert_matrix(wl, seed_off + l, role, e, dev)  # noqa: E731
        layers.append(quantize_layer(wl.hidden, wl.ffn, wl.n_experts, wl.top_k, fn, fmt=wl.fmt))
        routers.append(synthetic.router(wl, seed_off + l, dev))
    return layers, routers


def build_shared(B, wl, n_layers, dev, seed_off):
    """The shared expert of each layer of the stack (8-bit blocks)."""
    import synthetic
    return [B.SharedExpert(*[synthetic.shared_matrix(wl, seed_off + l, r, dev) for r in ("gate", "up", "down")])
            for l in range(n_layers)]


def run_workload(B, wl, layers, routers, steps, warmup, dev, world, seed_off, do_e2e=True):
    """Warm-up, CUDA-graph capture and the timed region for one workload,
    then its per-kernel times and roofline.  Returns the result dict."""
    import torch
    import torch.distributed as dist
    import synthetic
    T, H, K = wl.ntok, wl.hidden, wl.top_k
    L = len(layers)
    NX = 64 if T <= 64 else 4
    xs = [synthetic.activations(wl, seed_off + j, device=dev) for j in range(NX)]
    ws = B.Workspace.for_layer(layers[0], T)
    y = torch.empty((T, H), dtype=torch.float32, device=dev)
    shared = build_shared(B, wl, L, dev, seed_off) if wl.shared_ffn else None
    if shared:
        sws = shared[0].workspace(T, dev)
    torch.cuda.synchronize()

    def step(j):
        if shared:
            # the routed experts and the shared expert's FFN: one launch for
            # one token (the shared expert inside the one-token step), else
            # the routed kernels, then the shared expert's gate/up with the
            # requantization and its down mat-vec with the add into y
            B.moe_forward_shared(layers[j % L], shared[j % L], routers[j % L], xs[j % NX], ws, sws, y=y)
        else:
            B.moe_forward(layers[j % L], routers[j % L], xs[j % NX], ws, y=y)

    for j in range(warmup):
        step(j)
    torch.cuda.synchronize()
    status = B.moe_check_status(ws)
    if status != 0:
        raise SystemExit("device status %d after warm-up" % status)
    G = min(steps, 4 * L)
    stream = torch.cuda.Stream(device=dev)

    def capture(n_steps, first):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            step(first)  # make sure the stream has run the path once
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for j in range(n_steps):
                    step(first + j)
        return g

    g_main = capture(G, warmup)
    rem = steps % G
    g_rem = capture(rem, warmup) if rem else None
    reps = steps // G
    c0 = B.moe_launch_count()
    step(0)
    launches_per_step = B.moe_launch_count() - c0
    torch.cuda.synchronize()
    g_main.replay()  # untimed warm replay
    torch.cuda.synchronize()

    # ---- timed region
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g_main.replay()
            if g_rem is not None:
                g_rem.replay()
            e1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    status = B.moe_check_status(ws)
    if status != 0:
        raise SystemExit("device status %d after the timed region" % status)
    del g_main, g_rem

    # ---- per-kernel times: the same steps launched eagerly behind a spin
    # kernel (so the host has queued them all before the GPU starts them and
    # they run back to back), with an event after every library kernel
    n_tr = min(G, 2 * L) if T <= 64 else min(G, 4)
    per_kernel = {}
    for _ in range(3):
        tr = B.KernelTrace(capacity=n_tr * launches_per_step + 8)
        with torch.cuda.stream(stream):
            torch.cuda._sleep(int(4e7))
            with tr:
                for j in range(n_tr):
                    step(warmup + j)
            stream.synchronize()
        for name, v in tr.durations().items():
            per_kernel.setdefault(name, []).extend(v)
    # routing of the (layer, input) combinations the steps use: unique experts
    uniq = []
    for j in range(min(L * NX, 256 if T <= 64 else 8)):
        idx, _ = B.moe_route_topk(xs[j % NX], routers[j % L], K)
        uniq.append(len(set(idx.flatten().tolist())))
    unique_experts = sum(uniq) / len(uniq)
    kb = kernel_bytes(wl, unique_experts)
    total_ms = sum(sum(v) for v in per_kernel.values())
    shares = {n: {"avg_us": 1e3 * sum(v) / len(v), "share": sum(v) / total_ms,
                  "launches": len(v)} for n, v in per_kernel.items()}
    dom = max(shares, key=lambda n: shares[n]["share"])
    peak, peak_kind = measured_peaks()
    eager_s = shares[dom]["avg_us"] / 1e6
    if launches_per_step == 1 and len(shares) == 1:
        # one kernel per step: its average launch duration is the timed
        # region's time over its launches (the replayed launches overlap a
        # launch's start with the previous one's end, which the eager,
        # event-separated timing above does not)
        avg_s, dur_src = ms / 1e3 / steps, "timed region / launches"
    else:
        avg_s, dur_src = eager_s, "events around each launch, launched back to back"
    achieved = kb.get(dom, 0) / avg_s / 1e9
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_source": peak_kind,
                "algorithmic_bytes_per_launch": kb.get(dom, 0),
                "traffic": ncu_traffic(dom, wl.describe()),
                "launch_us": avg_s * 1e6, "launch_us_source": dur_src,
                "achieved_event_timed": kb.get(dom, 0) / eager_s / 1e9}
    step_bytes = sum(kb[n] for n in kb if n in shares)
    step_s = ms / 1e3 / steps
    res = {"workload": wl.describe(), "tokens_per_step": T, "steps": steps, "warmup": warmup,
           "ms_per_step": ms / steps, "value": job_rate(T * steps, world, ms), "unit": "tok/s",
           "layer_stack": L, "roofline": roofline, "step_hbm_gbs": step_bytes / step_s / 1e9,
           "step_hbm_frac": step_bytes / step_s / 1e9 / peak,
           "unique_experts_per_step": unique_experts, "kernels": shares,
           "launches_per_step": launches_per_step, "clocks": sampler.summary()}
    if wl.prefill:
        macs = T * K * 3 * H * wl.ffn
        gemm_s = sum(shares[n]["avg_us"] for n in ("prefill_gateup", "prefill_down") if n in shares) / 1e6
        res["int8_tops"] = {"value": 2 * macs / gemm_s / 1e12 if gemm_s else None,
                            "macs_per_step": macs, "kernels": ["prefill_gateup", "prefill_down"],
                            "tensor_pipe_pct": ncu_field("prefill_gateup", wl.describe(), "tensor_pipe_pct")}
    if T > 1:
        res["routing_histogram"] = routing_histogram(B, xs[0], routers[0], wl)

    # ---- end to end: the host-buffer entry point, copies inside the timed region.
    # Every step copies its x in from pinned host memory and its y out to pinned
    # host memory on the stream; the steps are replayed from CUDA graphs of
    # moe_forward_host calls, as a serving loop would drive them.
    if do_e2e and not wl.shared_ffn:  # the host-buffer entry point has no shared expert
        n_e2e = min(steps, 2000)
        xh = [xs[j % NX].cpu().pin_memory() for j in range(min(NX, n_e2e))]
        yh = torch.empty((T, H), dtype=torch.float32).pin_memory()

        def host_step(j):
            B.moe_forward_host(layers[j % L], routers[j % L], xh[j % len(xh)], yh, ws, stream=stream)

        def capture_host(n_steps):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                host_step(0)
                stream.synchronize()
                with torch.cuda.graph(g, stream=stream):
                    for j in range(n_steps):
                        host_step(j)
            return g

        Ge = min(n_e2e, 4 * L * len(xh))
        ge_main = capture_host(Ge)
        ge_rem = capture_host(n_e2e % Ge) if n_e2e % Ge else None
        with torch.cuda.stream(stream):
            ge_main.replay()
            stream.synchronize()
            if world > 1:
                dist.barrier()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(n_e2e // Ge):
                ge_main.replay()
            if ge_rem is not None:
                ge_rem.replay()
            a1.record(stream)
            stream.synchronize()
        del ge_main, ge_rem
        e_ms = max_over_ranks(a0.elapsed_time(a1), world, dev)
        res["e2e"] = {"value": job_rate(T * n_e2e, world, e_ms), "unit": "tok/s",
                      "h2d_bytes_per_step": T * H * 4, "d2h_bytes_per_step": T * H * 4,
                      "steps": n_e2e, "api": "moe_forward_host", "launch": "CUDA graph replay"}
    return res


# the other configurations measured in the same run (single GPU): the large
# layer at 8 tokens, the 30B-class layer at 1 and 16 tokens, and its
# 2048-token prefill
SUITE = ("large-b8", "30b", "30b-shared", "30b-b16", "30b-prefill")


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    rank, world, local = dist_env()
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    import bit_moe_b200 as B
    import synthetic
    from bit_moe_b200 import build
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    B.lib()

    wl = synthetic.WORKLOADS[args.workload]
    T, H, K = wl.ntok, wl.hidden, wl.top_k
    dev = torch.device("cuda", local)
    seed_off = 1000 * rank  # each replica draws its own layers and inputs

    def stack_for(w):
        per_step_guess = (min(w.n_experts, w.ntok * w.top_k) * w.expert_bytes) + w.n_experts * w.hidden * 4
        return args.layers if args.layers > 0 else stack_size(w, per_step_guess)

    # ---- headline workload: layer stack and inputs resident in HBM
    L = stack_for(wl)
    layers, routers = build_stack(B, wl, L, dev, seed_off)
    head = run_workload(B, wl, layers, routers, args.steps, args.warmup, dev, world, seed_off,
                        do_e2e=not args.no_e2e)

    # ---- the other configurations (one GPU only): each on its own stack,
    # the large layer's reused where the seeds agree
    suite = []
    if world == 1 and not args.no_suite and args.workload == "large":
        held = wl  # the workload whose layer stack is built
        for name in SUITE:
            w = synthetic.WORKLOADS[name]
            same = lambda a, b: (a.hidden, a.ffn, a.n_experts, a.seed, a.fmt) == (b.hidden, b.ffn, b.n_experts,  # noqa: E731
                                                                                 b.seed, b.fmt)
            if not same(w, held) or stack_for(w) > len(layers):
                del layers, routers
                torch.cuda.empty_cache()
                layers, routers = build_stack(B, w, stack_for(w), dev, seed_off)
                held = w
            suite.append(run_workload(B, w, layers, routers, max(args.steps, 20), max(args.warmup, 3), dev,
                                      world, seed_off, do_e2e=not args.no_e2e))
    del layers, routers
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(synthetic.WORKLOADS[args.workload])

    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8",
            "data": "synthetic", "config": workload_config(synthetic.WORKLOADS[args.workload], L),
            "roofline": head["roofline"], "cpu_baseline": cpu, "e2e": head.get("e2e"),
            "gpu_launches": head["launches_per_step"] * args.steps,
            "clocks": head["clocks"],
            "step_hbm_gbs": head["step_hbm_gbs"], "step_hbm_frac": head["step_hbm_frac"],
            "unique_experts_per_step": head["unique_experts_per_step"],
            "kernels": head["kernels"],
            "configs": suite,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
