"""Benchmark of the seed-decompress MoE decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--batch T] [--impl ours|reference]

A step is one decode step of T tokens (default 1) through a 45-layer stack of
seed-packed MoE layers (100 experts per layer, hidden 2048, expert
intermediate 1408, P=4, top-8 routing from N(0,1) logits): per layer routing,
gate/up + SiLU, down + weighted sum, then the RMS chaining into the next
layer, all through the library's C ABI (nslm_moe_stack_decode) captured in a
CUDA graph.  The 21.9 GB of packed experts stay resident in HBM; a token reads
1.75 GB of them, far more than the 126 MB L2, so no flush is needed.

The JSON line also carries the seed-GEMV sweep (packed-byte GB/s per expert
shape, rotating copies to defeat L2), a roofline object for the per-layer
decode FFN, the end-to-end number through the C ABI with host buffers, the
clocks seen during the timed region and the CPU oracle's time on a sample.
Extra objects, each skippable by its flag: one_layer_decode (one layer's
latency and HBM fraction), stack_batch8 (the same stack at 8 tokens a step,
--no-batch8), batched (the tcgen05 grouped GEMM layer at 64 and 512 tokens,
--no-batched), stack_p3c5 (the one-token stack in the 5-bit P=3 format,
--no-p3c5), host_experts (experts kept in pinned host memory behind the
device expert cache, one GPU only, --no-host-experts) and seed_search (the
seed/coefficient search, plain and importance-weighted, --no-search).
--profile runs one small case of a single kernel family for ncu and prints
no JSON line.

--impl reference times the CPU oracle (the plain C definition of the method)
on this host's cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))

# the sources the one-token decode kernel is compiled from: a traffic figure
# recorded under profiles/ is used only while their digest is unchanged
KERNEL_SOURCES = ("stack1.cu", "stack1.cuh", "chunk.cuh", "regen.cuh", "persist.cuh", "common.cuh", "moe.cuh")


def layer_record(path: str | None = None) -> dict:
    """The per-layer ncu record of the one-token kernel (profiles/
    ffn_decode_layer_traffic.txt): its integer fields, and whether its
    digest matches the kernel sources as they are now (the figures hold only
    then)."""
    path = path or os.path.join(ROOT, "profiles", "ffn_decode_layer_traffic.txt")
    rec = {}
    if os.path.exists(path):
        for ln in open(path):
            if ":" in ln and not ln.startswith("#"):
                key, val = ln.split(":", 1)
                rec[key.strip()] = val.split()[0] if val.split() else ""
    out = {"matches": bool(rec) and rec.get("kernel_sources_sha256") == kernel_sources_sha256()}
    for key in ("dram_bytes_per_layer_call", "warp_instructions_per_layer_call"):
        try:
            out[key] = int(rec[key])
        except (KeyError, ValueError):
            out[key] = None
    return out


def kernel_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "lfsr_seeded_moe_b200", "csrc", name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

E, HIDDEN, INTER, P, K_TOP, LAYERS = 100, 2048, 1408, 4, 8, 45
WORKLOAD = "45-layer seed-expert MoE decode: 100 experts/layer, hidden 2048, inter 1408, P=4, top-8"
METRIC = "MoE seed-FFN decode tokens/s"
GEMV_METRIC = "seed-GEMV packed-byte HBM GB/s (% of peak)"
GEMV_SHAPES = [(2048, 4096), (4096, 2048), (1408, 2048), (2048, 1408)]  # the expert-sized sweep
GEMV_SMALL = (512, 1024)  # the single small GEMV (P=4); L2-resident, so its % of HBM means little
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (context beside the measured copy peak)
FALLBACK_HBM_GBS = 6650.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def layer_packed_bytes_per_token(per_block: float = 4.5) -> int:
    """Packed bytes one token reads in one layer: 8 experts' gate, up and down
    fields (per_block bytes per 8-weight block: 4.5 for P=4, 4.375 for the
    5-bit P=3 format) plus an int32 exponent bias per row."""
    per_expert = 2 * (INTER * (HIDDEN // 8) * per_block + 4 * INTER) + (HIDDEN * (INTER // 8) * per_block + 4 * HIDDEN)
    return int(K_TOP * per_expert)


# ------------------------------------------------------------------ clocks

_POLLER = r"""
import sys, time
import pynvml as nv
uuid, index, period = sys.argv[1], int(sys.argv[2]), float(sys.argv[3])
nv.nvmlInit()
try:
    h = nv.nvmlDeviceGetHandleByUUID(uuid) if uuid else nv.nvmlDeviceGetHandleByIndex(index)
except nv.NVMLError:
    h = nv.nvmlDeviceGetHandleByIndex(index)
try:
    mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
except nv.NVMLError:
    mx = "[N/A]"
bits = (0x8, 0x40, 0x20, 0x4)
print("ready", flush=True)
while True:
    try:
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        flags = ", ".join("Active" if rs & b else "Not Active" for b in bits)
        print(f"{time.monotonic():.6f}|{index}, {sm}, {mx}, {pw:.1f}, {rs:#x}, {flags}", flush=True)
    except nv.NVMLError:
        pass
    time.sleep(period)
"""


class ClockSampler:
    """Samples SM clocks and throttle reasons while the timed region runs.

    A child process polls NVML every 2 ms (a process of its own, so that the
    timed loop, which holds the interpreter lock, cannot starve it) on the GPU
    that CUDA device `dev` is (matched by UUID, since CUDA and NVML may number
    GPUs differently) and stamps each sample with the monotonic clock; only
    samples inside the marked window (mark_start / mark_end around the timed
    region) are kept.  Without NVML, nvidia-smi runs at its 20 ms interval.
    Every sample is kept as one CSV row in nvidia-smi's field order."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML reason bits, in the order of the last four fields
    BITS = (0x8, 0x40, 0x20, 0x4)

    def __init__(self, gpu_index: int, uuid: str | None = None, period_s: float = 0.002):
        self.gpu = gpu_index
        self.uuid = uuid
        self.period = period_s
        self.proc = None
        self.thread = None
        self.stamped = []   # (monotonic time, row) from the NVML poller
        self.lines = []     # rows kept for the summary
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", _POLLER, self.uuid or "", str(self.gpu), str(self.period)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            if self.proc.stdout.readline().strip() != "ready":
                raise OSError("no NVML poller")
            self.thread = threading.Thread(target=self._read_stamped, daemon=True)
            self.thread.start()
            return self
        except OSError:
            if self.proc is not None:
                self.proc.kill()
            self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def _read_stamped(self):
        for line in self.proc.stdout:
            t, _, row = line.strip().partition("|")
            try:
                self.stamped.append((float(t), row))
            except ValueError:
                pass

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(2 * self.period)  # the samples of the window's last moments
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        self.keep_window()

    def keep_window(self):
        """Keep the stamped samples taken inside [mark_start, mark_end]."""
        if self.stamped:
            t0 = self.t0 if self.t0 is not None else float("-inf")
            t1 = self.t1 if self.t1 is not None else float("inf")
            self.lines.extend(row for t, row in self.stamped if t0 <= t <= t1)
            self.stamped = []

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def device_uuid(torch, dev) -> str | None:
    """NVML's name of the GPU behind CUDA device `dev` ("GPU-<uuid>")."""
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return None


# --------------------------------------------------------------- oracle leg

def oracle_layer_seconds(n_layers: int, T: int = 1, seed_tag: int = 0):
    """Time the CPU oracle on n_layers decode layers of T tokens (routed experts only)."""
    import numpy as np

    from lfsr_seeded_moe_b200 import synth
    from oracle import oracle as O

    total = 0.0
    for li in range(n_layers):
        logits = synth.router_logits((4, li, seed_tag), T, E).numpy()
        ids, w = O.route_topk(logits, K_TOP)
        experts = sorted(set(int(e) for e in ids.reshape(-1)))
        # a compact stack with only the routed experts, drawn on the host
        remap = {e: i for i, e in enumerate(experts)}
        sl = [synth.expert_slice(li, e, E, HIDDEN, INTER, P, config=4) for e in experts]

        def stack(name):
            class _S:
                pass
            s = _S()
            parts = [getattr(x, name).numpy() for x in sl]
            s.seeds = np.concatenate([q.seeds for q in parts])
            s.coefs = np.concatenate([q.coefs for q in parts])
            s.codes = np.concatenate([q.codes for q in parts])
            s.exp_bias = np.concatenate([q.exp_bias for q in parts])
            s.P = P
            return s

        g, u, d = stack("gate"), stack("up"), stack("down")
        x = synth.bf16_bits(synth.activations((4, seed_tag), T, HIDDEN)).numpy().view(np.uint16)
        ids_c = np.vectorize(lambda e: remap[int(e)])(ids).astype(np.int32)
        t0 = time.perf_counter()
        O.moe_ffn(g, u, d, len(experts), HIDDEN, INTER, x, ids_c, w, mode=0)
        total += time.perf_counter() - t0
    return total


def workload_config(T: int, world: int) -> dict:
    """The workload both arms report (the same dict, key for key)."""
    per_expert = layer_packed_bytes_per_token() // K_TOP
    return {"workload": WORKLOAD, "batch_tokens": T, "layers": LAYERS, "experts": E,
            "hidden": HIDDEN, "inter": INTER, "P": P, "top_k": K_TOP,
            "packed_GB_resident": round(LAYERS * E * per_expert / 1e9, 3),
            "l2": "inputs larger than L2 (1.75 GB of weights read per token)",
            "parallelism": f"replicas x{world}"}


def cpu_model() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_gemvs(O, synth, np):
    """The single small GEMV (512 x 1024, P=4) and the expert-sized sweep
    (P=4 and P=3) on the oracle: us, weights/s and packed-GB/s equivalent."""
    out = []
    for Pv, (N, K) in [(4, GEMV_SMALL)] + [(Pv, nk) for Pv in (4, 3) for nk in GEMV_SHAPES]:
        m = synth.seed_matrix(N, K, Pv, (11, N, K, Pv)).numpy()
        x = synth.bf16_bits(synth.activations((11,), 1, K)).numpy().view(np.uint16)
        reps = 4 if N * K < 2 ** 21 else 1
        t0 = time.perf_counter()
        for _ in range(reps):
            O.seed_matvec(m, x)
        t = (time.perf_counter() - t0) / reps
        out.append({"P": Pv, "N": N, "K": K, "us": round(t * 1e6, 1), "weights_per_s": round(N * K / t, 1),
                    "packed_GB_s": round(O.packed_bytes(N, K, Pv) / t / 1e9, 4)})
    return out


def cpu_baseline(budget_s: float = 12.0, T: int = 1):
    """The oracle timed on this host's cores, with all threads and with one:
    the seed GEMVs (the 512 x 1024 GEMV and the expert-sized sweep), one
    decode layer (one token) and the 45-layer stack (one token, a sample of
    layers scaled to 45).  The headline value is the stack's tokens/s on all
    cores."""
    import numpy as np

    from lfsr_seeded_moe_b200 import synth
    from oracle import oracle as O

    all_cores = O.threads_used()
    runs = {}
    try:
        for threads, share in ((all_cores, 0.6), (1, 0.4)):
            O.lib().omp_set_num_threads(threads)
            gemv = _oracle_gemvs(O, synth, np)
            t1 = oracle_layer_seconds(1, T, seed_tag=1)
            n = max(1, min(LAYERS, int(share * budget_s / max(t1, 1e-3))))
            t = oracle_layer_seconds(n, T, seed_tag=2) if n > 1 else t1
            per_layer = t / n
            runs[threads] = {
                "threads": threads, "gemv": gemv,
                "one_layer": {"us": round(t1 * 1e6, 1), "tokens_per_s": round(T / t1, 3),
                              "weights_per_s": round(K_TOP * 3 * HIDDEN * INTER * T / t1, 1),
                              "packed_GB_s": round(layer_packed_bytes_per_token() / t1 / 1e9, 4)},
                "stack": {"tokens_per_s": T / (per_layer * LAYERS), "layers_timed": n,
                          "s_per_layer": round(per_layer, 4),
                          "packed_GB_s": round(layer_packed_bytes_per_token() / per_layer / 1e9, 4)},
            }
    finally:
        O.lib().omp_set_num_threads(all_cores)
    top = runs[all_cores]["stack"]
    return {"value": top["tokens_per_s"], "unit": "tokens/s", "cores": all_cores, "kind": "oracle",
            "nproc": os.cpu_count(), "cpu_model": cpu_model(),
            "sample": f"{top['layers_timed']} layer(s) x {T} token(s) of the 45-layer stack on all "
                      f"{all_cores} threads (oracle fp64, routed experts only), scaled to 45 layers; "
                      f"per-config figures on all threads and on one in 'all_cores' / 'one_core'",
            "all_cores": runs[all_cores], "one_core": runs[1]}


def run_reference(args):
    """The reference arm: the CPU oracle (the plain C definition of the method)
    on this host's cores.  Each step is a bounded sample of the workload: one
    layer of the 45-layer stack for the step's tokens (a different layer and
    routing each step).  ms_per_step is that measured sample; value scales it to
    the whole stack's tokens/s."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import oracle as O

    T = args.batch
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    for i in range(args.warmup):
        oracle_layer_seconds(1, T, seed_tag=100 + i)
    times = [oracle_layer_seconds(1, T, seed_tag=200 + i) for i in range(args.steps)]
    per_layer = sum(times) / len(times)
    tok_s = T / (per_layer * LAYERS)
    sample = (f"each of {args.steps} step(s): one decode layer of the 45-layer stack for {T} token(s) on the "
              f"oracle (fp64, {O.threads_used()} threads); tokens/s = tokens / (45 x the mean layer time)")
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per_layer * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded SplitMix64 fields)",
        "config": workload_config(T, world),
        "step": "one of the stack's 45 layers (a bounded sample); ms_per_step is its measured time",
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": O.threads_used(), "kind": "oracle",
                         "nproc": os.cpu_count(), "cpu_model": cpu_model(), "sample": sample},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def slowest_rank_time(elapsed_s: float, world: int, device) -> float:
    """The timed region's duration as the maximum over the ranks of the job
    (one process per GPU; every rank calls this at the same point)."""
    if world <= 1:
        return elapsed_s
    import torch
    import torch.distributed as dist
    t = torch.tensor([elapsed_s], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, tokens_per_step: int, elapsed_s: float) -> float:
    """Whole-job tokens/s: every rank decodes its own tokens (replicas)."""
    return world * steps * tokens_per_step / elapsed_s


# ------------------------------------------------------------------- GPU leg

def gemv_sweep(torch, nslm, synth, dev, hbm, shapes=None):
    """The single small GEMV (512 x 1024, P=4) and the expert-sized sweep for
    P=4, P=3 and the 5-bit P=3 format (35), batch 1.  Each shape is timed over
    rotating weight copies in one CUDA graph (more than 4x L2 where 400 copies
    reach it; the small GEMV's copies stay largely in L2): the cold (HBM)
    figures.  The warm figures repeat one copy, which then sits in L2.
    `shapes` ([(N, K), ...]) replaces the whole list, small GEMV included."""
    out = []
    if shapes:
        cases = [(Pv, nk) for Pv in (4, 3, 35) for nk in shapes]
    else:
        cases = [(4, GEMV_SMALL)] + [(Pv, nk) for Pv in (4, 3, 35) for nk in GEMV_SHAPES]
    for Pv, (N, K) in cases:
        m0 = synth.seed_matrix(N, K, Pv, (11, N, K, Pv), device=dev)
        nbytes = m0.packed_bytes()
        ncopy = min(400, max(2, int(4 * 126e6 // nbytes) + 1))
        mats = [synth.seed_matrix(N, K, Pv, (11, N, K, Pv, c), device=dev) for c in range(ncopy)]
        structs = [nslm.matrix(m) for m in mats]
        x = synth.activations((11,), 1, K).to(dev)
        y = torch.empty(1, N, device=dev)
        nslm.nslm_seed_gemv(structs[0], x, 1, y)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for c in range(ncopy):
                nslm.nslm_seed_gemv(structs[c], x, 1, y)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) * 1e-3 / (reps * ncopy)
        gbs = nbytes / t / 1e9
        # the same chain with NSLM_GEMV_FIELDS_READY (no kernel writes the
        # weights, so each GEMV's first field copies overlap its predecessor)
        gf = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gf):
            for c in range(ncopy):
                nslm.nslm_seed_gemv_flags(structs[c], x, 1, y, nslm.NSLM_GEMV_FIELDS_READY)
        for _ in range(3):
            gf.replay()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            gf.replay()
        e1.record()
        torch.cuda.synchronize()
        tf = e0.elapsed_time(e1) * 1e-3 / (reps * ncopy)
        nwarm = 100
        gw = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gw):
            for _ in range(nwarm):
                nslm.nslm_seed_gemv(structs[0], x, 1, y)
        for _ in range(3):
            gw.replay()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            gw.replay()
        e1.record()
        torch.cuda.synchronize()
        tw = e0.elapsed_time(e1) * 1e-3 / (reps * nwarm)
        out.append({"P": Pv, "N": N, "K": K, "us": round(t * 1e6, 3), "GB_s": round(gbs, 1),
                    "pct_of_hbm": round(100 * gbs / hbm, 2),
                    "pct_of_nominal_8TBs": round(100 * gbs / NOMINAL_HBM_GBS, 2), "weights_per_s": N * K / t,
                    "fields_ready_us": round(tf * 1e6, 3), "fields_ready_GB_s": round(nbytes / tf / 1e9, 1),
                    "fields_ready_pct_of_hbm": round(100 * nbytes / tf / 1e9 / hbm, 2),
                    "rotated_bytes": nbytes * ncopy, "rotation_below_4x_l2": nbytes * ncopy < 4 * 126e6,
                    "warm_L2_us": round(tw * 1e6, 3), "warm_L2_GB_s": round(nbytes / tw / 1e9, 1)})
        del g, gf, gw, mats, structs
        torch.cuda.empty_cache()
    return out


def batched_sweep(torch, nslm, synth, dev, hbm, bf16_peak):
    """Batched MoE layer on the tensor-core path: 100 experts, 2048/1408, P=3, top-8."""
    Pb, nl = 3, 4
    layers = [synth.moe_layer(l, E, HIDDEN, INTER, Pb, device=dev, config=3) for l in range(nl)]
    per_expert = 2 * (INTER * (HIDDEN // 8) * 4 + 4 * INTER) + (HIDDEN * (INTER // 8) * 4 + 4 * HIDDEN)
    out = []
    for T in (64, 512):
        for zipf in (None, 1.1):
            logits = synth.router_logits((3, T, zipf is not None), T, E, zipf).to(dev)
            ids = torch.empty(T, K_TOP, dtype=torch.int32, device=dev)
            w = torch.empty(T, K_TOP, device=dev)
            nslm.nslm_moe_route_topk(logits, T, E, K_TOP, ids, w)
            x = synth.activations((3, T), T, HIDDEN).to(dev)
            y = torch.empty(T, HIDDEN, device=dev)
            wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, E, HIDDEN, INTER, K_TOP)
            ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
            st = [(nslm.matrix(L.gate), nslm.matrix(L.up), nslm.matrix(L.down)) for L in layers]
            nslm.nslm_moe_seed_ffn(*st[0], E, x, ids, w, T, K_TOP, y, ws, wsb)
            torch.cuda.synchronize()
            reps = 2 * nl
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(reps):
                    nslm.nslm_moe_seed_ffn(*st[i % nl], E, x, ids, w, T, K_TOP, y, ws, wsb)
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) * 1e-3 / (2 * reps)
            status = int(ws[:4].view(torch.int32).item())
            uniq = len(set(ids.cpu().numpy().reshape(-1).tolist()))
            nbytes = uniq * per_expert
            flops = 2.0 * T * K_TOP * 3 * INTER * HIDDEN
            out.append({"T": T, "routing": "zipf1.1" if zipf else "uniform", "experts_touched": uniq,
                        "us_per_layer": round(t * 1e6, 2), "tokens_per_s_per_layer": round(T / t, 1),
                        "packed_GB_s": round(nbytes / t / 1e9, 1), "pct_of_hbm": round(100 * nbytes / t / 1e9 / hbm, 2),
                        "mma_TFLOP_s": round(flops / t / 1e12, 1),
                        "pct_of_bf16_peak": round(100 * flops / t / 1e12 / bf16_peak, 2) if bf16_peak else None,
                        "status": status})
            del g
    del layers
    torch.cuda.empty_cache()
    return out


class _Encoded:
    """Device streams of an N x K packed matrix for the seed search to fill."""

    def __init__(self, torch, dev, N, K, P, bias):
        nb = K // 8
        self.N, self.K, self.P = N, K, P
        self.seeds = torch.empty(N, nb, dtype=torch.int16, device=dev)
        self.coefs = torch.empty(N, nb, dtype=torch.int16, device=dev)
        self.codes = torch.empty(N, nb // 2, dtype=torch.uint8, device=dev) if P == 4 else None
        self.exp_bias = torch.full((N,), bias, dtype=torch.int32, device=dev)


def stack_batch_leg(torch, nslm, synth, dev, arr, hbm, T: int, steps: int, rank: int):
    """The same resident 45-layer stack decoding T tokens per step (one CUDA
    graph per step, 8 distinct step inputs cycled).  Packed bytes per step
    count each layer's distinct routed experts once (tokens share them)."""
    S = 8
    logits = [torch.stack([synth.router_logits((4, l, rank, s, T), T, E) for l in range(LAYERS)]).to(dev).contiguous()
              for s in range(S)]
    xs = [synth.activations((4, rank, s, T), T, HIDDEN).to(dev).contiguous() for s in range(S)]
    y = torch.empty(T, HIDDEN, device=dev)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_STACK, T, E, HIDDEN, INTER, K_TOP, LAYERS)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    nslm.nslm_moe_stack_decode(arr, LAYERS, E, K_TOP, logits[0], xs[0], T, y, ws, wsb)
    launches = nslm.nslm_last_launch_count()
    torch.cuda.synchronize()
    graphs = []
    for s in range(S):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            nslm.nslm_moe_stack_decode(arr, LAYERS, E, K_TOP, logits[s], xs[s], T, y, ws, wsb)
        graphs.append(g)
    for i in range(3):
        graphs[i % S].replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        graphs[i % S].replay()
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) * 1e-3 / steps
    status = int(ws[:4].view(torch.int32).item())
    # distinct experts per layer from the same top-k (N(0,1) logits: no ties)
    per_expert = layer_packed_bytes_per_token() / K_TOP
    step_bytes = [sum(len(set(lg[l].topk(K_TOP, dim=-1).indices.reshape(-1).tolist())) for l in range(LAYERS))
                  * per_expert for lg in logits]
    mean_bytes = sum(step_bytes[i % S] for i in range(steps)) / steps
    graphs.clear()
    return {"batch_tokens": T, "value": round(T / t, 2), "unit": "tokens/s", "ms_per_step": round(t * 1e3, 4),
            "steps": steps, "status": status, "gpu_launches_per_step": launches,
            "packed_GB_per_step": round(mean_bytes / 1e9, 3),
            "hbm_frac": round(mean_bytes / t / 1e9 / hbm, 4),
            "note": "one cooperative launch for all 45 layers (plus the routing launch); inputs > L2"}


def stack_p3c5_leg(torch, nslm, synth, dev, hbm, steps: int, rank: int):
    """The 45-layer one-token stack with every expert in the 5-bit P=3 format
    (4.375 bits per weight), on the same persistent kernel, 8 cycled inputs."""
    Pf, S = nslm.NSLM_P3C5, 8
    layers = [synth.moe_layer(l, E, HIDDEN, INTER, Pf, device=dev, config=5) for l in range(LAYERS)]
    arr = nslm.moe_layers([(L.gate, L.up, L.down) for L in layers])
    logits = [torch.stack([synth.router_logits((5, l, rank, s), 1, E) for l in range(LAYERS)]).to(dev).contiguous()
              for s in range(S)]
    xs = [synth.activations((5, rank, s), 1, HIDDEN).to(dev).contiguous() for s in range(S)]
    y = torch.empty(1, HIDDEN, device=dev)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_STACK, 1, E, HIDDEN, INTER, K_TOP, LAYERS)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    graphs = []
    for s in range(S):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            nslm.nslm_moe_stack_decode(arr, LAYERS, E, K_TOP, logits[s], xs[s], 1, y, ws, wsb)
        graphs.append(g)
    for i in range(3):
        graphs[i % S].replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        graphs[i % S].replay()
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) * 1e-3 / steps
    status = int(ws[:4].view(torch.int32).item())
    nbytes = LAYERS * layer_packed_bytes_per_token(4.375)
    graphs.clear()
    del layers, arr
    torch.cuda.empty_cache()
    return {"format": "P=3 with 5-bit coefficients (4.375 bits per weight)", "batch_tokens": 1,
            "value": round(1.0 / t, 2), "unit": "tokens/s", "ms_per_step": round(t * 1e3, 4), "steps": steps,
            "status": status, "packed_GB_per_step": round(nbytes / 1e9, 3),
            "hbm_frac": round(nbytes / t / 1e9 / hbm, 4),
            "note": "one cooperative launch for all 45 layers (plus the routing launch); inputs > L2"}


def host_experts_leg(torch, nslm, synth, dev, n_layers: int = 8, slots: int = 400, tokens: int = 32):
    """One-token decode with the routed experts in pinned host memory behind the
    VRAM expert cache (LRU, copies by the device from host memory): per token and
    layer, routing + cache fetch + the FFN on the cache.  8 layers x 100 experts
    (3.9 GB pinned) behind 400 slots, so about half the experts fit."""
    def pinned(m):
        return synth.SeedMatrix(m.seeds.pin_memory(), m.coefs.pin_memory(), m.codes.pin_memory(),
                                m.exp_bias.pin_memory(), m.rows, m.K, m.P, m.n_experts)

    def empty(rows, K):
        nb = K // 8
        return synth.SeedMatrix(torch.zeros(slots * rows, nb, dtype=torch.int16, device=dev),
                                torch.zeros(slots * rows, nb, dtype=torch.int16, device=dev),
                                torch.zeros(slots * rows, nb // 2, dtype=torch.uint8, device=dev),
                                torch.zeros(slots * rows, dtype=torch.int32, device=dev), rows, K, P, slots)

    host = []
    for l in range(n_layers):
        m = synth.moe_layer(l, E, HIDDEN, INTER, P, config=4)
        host.append(tuple(pinned(getattr(m, n)) for n in ("gate", "up", "down")))
    cache = (empty(INTER, HIDDEN), empty(INTER, HIDDEN), empty(HIDDEN, INTER))
    state = torch.zeros(nslm.nslm_expert_cache_state_bytes(slots), dtype=torch.uint8, device=dev)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, 1, slots, HIDDEN, INTER, K_TOP)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    warm = 16
    logits = [[synth.router_logits((4, l, 0, t), 1, E).to(dev) for l in range(n_layers)] for t in range(warm + tokens)]
    x = synth.activations((4, 0, 0), 1, HIDDEN).to(dev)
    ids = torch.empty(1, K_TOP, dtype=torch.int32, device=dev)
    w = torch.empty(1, K_TOP, device=dev)
    sl = torch.empty(1, K_TOP, dtype=torch.int32, device=dev)
    y = torch.empty(1, HIDDEN, device=dev)

    def token(t):
        for l in range(n_layers):
            nslm.nslm_moe_route_topk(logits[t][l], 1, E, K_TOP, ids, w)
            nslm.nslm_expert_cache_fetch(host[l], E, l, cache, slots, state, ids, 1, K_TOP, sl)
            nslm.nslm_moe_seed_ffn(cache[0], cache[1], cache[2], slots, x, sl, w, 1, K_TOP, y, ws, wsb)

    for t in range(warm):
        token(t)
    torch.cuda.synchronize()
    st0 = state[:16].view(torch.int32).cpu().tolist()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for t in range(warm, warm + tokens):
        token(t)
    e1.record()
    torch.cuda.synchronize()
    st1 = state[:16].view(torch.int32).cpu().tolist()
    dt = e0.elapsed_time(e1) * 1e-3
    hits, miss = st1[2] - st0[2], st1[3] - st0[3]
    per_expert = layer_packed_bytes_per_token() / K_TOP
    return {"workload": f"{n_layers} layers x {E} experts (P=4, 2048/1408) in pinned host memory, "
                        f"{slots}-slot VRAM expert cache, one token per step",
            "tokens_per_s": round(tokens / dt, 1), "ms_per_token": round(dt / tokens * 1e3, 3),
            "hit_rate": round(hits / max(1, hits + miss), 3), "misses_per_token": round(miss / tokens, 2),
            "copy_GB_per_s": round(miss * per_expert / dt / 1e9, 1)}


def search_leg(torch, nslm, dev, with_cpu: bool):
    """Seed search (the encoder) over all 65,535 seeds x 16 codes: GPU blocks/s
    on a 64 x 2048 fp32 matrix (16,384 blocks, P=4), and the oracle's time per
    block on two of them (one host core)."""
    N, K, Pv = 64, 2048, 4
    g = torch.Generator().manual_seed(0x5EED)
    w = (torch.randn(N, K, generator=g) * 4.0).to(dev)
    nslm.nslm_seed_search(w[:2], _Encoded(torch, dev, 2, K, Pv, -12), 1, 65535)  # warm-up
    out = _Encoded(torch, dev, N, K, Pv, -12)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    nslm.nslm_seed_search(w, out, 1, 65535)
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) * 1e-3
    nblk = N * (K // 8)
    # activation-weighted search: importances = mean squares of N(0,1)-like activations
    imp = (torch.rand(K, generator=g) * 2.0).to(dev)
    e0.record()
    nslm.nslm_seed_search(w, out, 1, 65535, imp=imp)
    e1.record()
    torch.cuda.synchronize()
    tw = e0.elapsed_time(e1) * 1e-3
    res = {"workload": "seed search of a 64 x 2048 fp32 matrix (16,384 blocks, P=4) over all 65,535 seeds x 16 codes",
           "gpu_blocks_per_s": round(nblk / t, 1), "gpu_s": round(t, 4),
           "candidates_per_s": nblk * 65535 * 16 / t,
           "gpu_blocks_per_s_weighted": round(nblk / tw, 1)}
    if with_cpu:
        from oracle import oracle as O
        wh = w[:1, :16].double().cpu().numpy()
        t0 = time.time()
        for b in range(2):
            O.search_block(wh[0, 8 * b:8 * b + 8], Pv, -12, 1, 65535)
        cpu = (time.time() - t0) / 2
        res["oracle_s_per_block_one_core"] = round(cpu, 4)
        res["gpu_vs_one_core"] = round(cpu * nblk / t, 1)
    return res


def anatomy(reps: int):
    """Per-layer anatomy of the one-token 45-layer launch from the trace build
    (`python -m lfsr_seeded_moe_b200.build --trace`; loaded here through
    NSLM_LIB_VARIANT=trace): medians over the middle layers of the global-timer
    stamps at each CTA's phase boundaries, in microseconds.  Prints one JSON
    line.  The trace build adds two block barriers a layer, so its layer time
    runs slightly above the default build's."""
    os.environ.setdefault("NSLM_LIB_VARIANT", "trace")
    import numpy as np
    import torch

    from lfsr_seeded_moe_b200 import nslm, synth

    if not nslm.LIB_PATH.endswith(os.path.join("trace", "libnslm.so")):
        raise SystemExit(f"--profile anatomy needs the trace build, loaded {nslm.LIB_PATH}")
    dev = torch.device("cuda", 0)
    layers = [synth.moe_layer(l, E, HIDDEN, INTER, 4, device=dev, config=4) for l in range(LAYERS)]
    arr = nslm.moe_layers([(m.gate, m.up, m.down) for m in layers])
    lg = torch.stack([synth.router_logits((4, l, 0, 0), 1, E) for l in range(LAYERS)]).to(dev).contiguous()
    x = synth.activations((4, 0, 0), 1, HIDDEN).to(dev).contiguous()
    y = torch.empty(1, HIDDEN, device=dev)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_STACK, 1, E, HIDDEN, INTER, K_TOP, LAYERS)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    for _ in range(max(2, reps)):
        nslm.nslm_moe_stack_decode(arr, LAYERS, E, K_TOP, lg, x, 1, y, ws, wsb)
    torch.cuda.synchronize()
    assert nslm.nslm_device_status(ws) == nslm.NSLM_OK
    t = nslm.nslm_debug_stack_trace().astype(np.float64) / 1e3  # us
    G = torch.cuda.get_device_properties(dev).multi_processor_count
    t = t[:, :G, :LAYERS]
    full = slice(0, max(1, G - 2))  # CTAs with a full share of output rows
    med = lambda a: float(np.median(a))
    rows = {}
    for l in range(2, LAYERS - 2):
        s0, s1, s2, s3, s4, s5, s6 = (t[k, :, l] for k in range(7))
        seg = {
            "stage_x": med(s1 - s0),
            "phase_A_median_cta": med(s2 - s1),
            "phase_A_tail": float(np.max(s2)) - med(s2),
            "barrier_after_last_arrival": med(s3) - float(np.max(s2)),
            "stage_h": med(s5 - s3),
            "phase_B_tasks": med((s6 - s5)[full]),
            "row_sums_and_y_stores": med((s4 - s6)[full]),
            "phase_B_tail": float(np.max(s4)) - med(s4),
            "phase_B_end_to_next_layer": med(t[0, :, l + 1] - s4),
            "layer": med(t[0, :, l + 1] - s0),
        }
        for k, v in seg.items():
            rows.setdefault(k, []).append(v)
    out = {"workload": "45-layer one-token decode stack, 100 experts, 2048/1408, P=4, top-8 (trace build)",
           "unit": "us", "layers_used": f"2..{LAYERS - 3}", "ctas": G}
    for k, v in rows.items():
        out[k] = round(float(np.median(v)), 2)
    lat = np.array([t[2, :, l] - np.median(t[2, :, l]) for l in range(2, LAYERS - 2)]).mean(0)
    out["phase_A_latest_ctas"] = {int(c): round(float(lat[c]), 2) for c in np.argsort(-lat)[:6]}
    print(json.dumps(out))


def profile_workload(kind: str, reps: int):
    """A small fixed workload for ncu captures (no timing, no JSON): `reps`
    calls of one decode layer (T=1 or T=8, P=4; T=1 in the 5-bit format), of
    one batched layer (T=512, P=3),
    of one seed GEMV (2048 x 4096, P=4) or of the seed search of a 16 x 256
    fp32 matrix over all seeds."""
    import torch

    from lfsr_seeded_moe_b200 import nslm, synth

    dev = torch.device("cuda", 0)
    if kind == "search":
        g = torch.Generator().manual_seed(0x5EED)
        w = (torch.randn(16, 256, generator=g) * 4.0).to(dev)
        out = _Encoded(torch, dev, 16, 256, 4, -12)
        for _ in range(reps):
            nslm.nslm_seed_search(w, out, 1, 65535)
        torch.cuda.synchronize()
        return
    if kind == "gemv":
        m = synth.seed_matrix(2048, 4096, 4, (11, 2048, 4096, 4), device=dev)
        x = synth.activations((11,), 1, 4096).to(dev)
        y = torch.empty(1, 2048, device=dev)
        for _ in range(reps):
            nslm.nslm_seed_gemv(nslm.matrix(m), x, 1, y)
        torch.cuda.synchronize()
        return
    T, Pv, cfg = {"layer": (1, 4, 2), "layer8": (8, 4, 2), "layer_p3c5": (1, nslm.NSLM_P3C5, 2)}.get(kind, (512, 3, 3))
    L = synth.moe_layer(0, E, HIDDEN, INTER, Pv, device=dev, config=cfg)
    logits = synth.router_logits((cfg, T), T, E).to(dev)
    ids = torch.empty(T, K_TOP, dtype=torch.int32, device=dev)
    w = torch.empty(T, K_TOP, device=dev)
    nslm.nslm_moe_route_topk(logits, T, E, K_TOP, ids, w)
    x = synth.activations((cfg, T), T, HIDDEN).to(dev)
    y = torch.empty(T, HIDDEN, device=dev)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, E, HIDDEN, INTER, K_TOP)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    for _ in range(reps):
        nslm.nslm_moe_seed_ffn(L.gate, L.up, L.down, E, x, ids, w, T, K_TOP, y, ws, wsb)
    torch.cuda.synchronize()
    if int(ws[:4].view(torch.int32).item()) != 0 and T > 8:
        raise SystemExit("batched layer reported a non-zero status")


def _gemv_shapes(text: str):
    """'8192x8192,2048x4096' -> [(8192, 8192), (2048, 4096)]."""
    out = []
    for part in text.split(","):
        n, k = part.lower().split("x")
        out.append((int(n), int(k)))
    if not out or any(n < 1 or k < 8 or k % 8 for n, k in out):
        raise argparse.ArgumentTypeError("shapes are NxK with N >= 1 and K a positive multiple of 8")
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--batch", type=int, default=1, help="decode tokens per step (1..8)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-gemv", action="store_true")
    ap.add_argument("--gemv-shapes", type=_gemv_shapes, default=None,
                    help="NxK[,NxK...]: the GEMV leg's shapes instead of its default sweep")
    ap.add_argument("--no-batched", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-search", action="store_true")
    ap.add_argument("--no-batch8", action="store_true", help="skip the 8-token stack leg")
    ap.add_argument("--no-host-experts", action="store_true", help="skip the host-memory expert cache leg")
    ap.add_argument("--no-p3c5", action="store_true", help="skip the 5-bit P=3 stack leg")
    ap.add_argument("--profile", choices=["layer", "layer8", "layer_p3c5", "batched", "gemv", "search", "anatomy"],
                    help="run a small fixed workload for an ncu capture and exit")
    args = ap.parse_args()
    if args.profile == "anatomy":
        return anatomy(args.steps)
    if args.profile:
        return profile_workload(args.profile, args.steps)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    from lfsr_seeded_moe_b200 import nslm, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    hbm, peak_kind = peaks()
    T = args.batch

    # --- resident expert stack (each rank holds its own replica)
    layers = [synth.moe_layer(l, E, HIDDEN, INTER, P, device=dev, config=4) for l in range(LAYERS)]
    arr = nslm.moe_layers([(L.gate, L.up, L.down) for L in layers])
    S = 8  # distinct step inputs, cycled
    logits = [torch.stack([synth.router_logits((4, l, rank, s), T, E) for l in range(LAYERS)]).to(dev).contiguous()
              for s in range(S)]
    xs = [synth.activations((4, rank, s), T, HIDDEN).to(dev).contiguous() for s in range(S)]
    y = torch.empty(T, HIDDEN, device=dev)
    wsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_STACK, T, E, HIDDEN, INTER, K_TOP, LAYERS)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)

    cs = torch.cuda.Stream()
    graphs = []
    with torch.cuda.stream(cs):
        nslm.nslm_moe_stack_decode(arr, LAYERS, E, K_TOP, logits[0], xs[0], T, y, ws, wsb, stream=cs)
        launches_per_step = nslm.nslm_last_launch_count()
    torch.cuda.synchronize()
    for s in range(S):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            nslm.nslm_moe_stack_decode(arr, LAYERS, E, K_TOP, logits[s], xs[s], T, y, ws, wsb)
        graphs.append(g)

    for i in range(max(3, args.warmup)):
        graphs[i % S].replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if dev.index is not None else 0, device_uuid(torch, dev)) as clk:
        torch.cuda.synchronize()
        clk.mark_start()
        e0.record()
        for i in range(args.steps):
            graphs[i % S].replay()
        e1.record()
        torch.cuda.synchronize()
        clk.mark_end()
    if world > 1:
        dist.barrier()
    elapsed = slowest_rank_time(e0.elapsed_time(e1) * 1e-3, world, dev)
    value = job_throughput(world, args.steps, T, elapsed)

    # --- end to end through the C ABI: pinned host inputs in, result out, every step
    hx = [x.cpu().pin_memory() for x in xs]
    hl = [lg.cpu().pin_memory() for lg in logits]
    hy = torch.empty(T, HIDDEN, dtype=torch.float32).pin_memory()
    dx = torch.empty_like(xs[0])
    dl = torch.empty_like(logits[0])
    h2d = hx[0].numel() * hx[0].element_size() + hl[0].numel() * hl[0].element_size()
    d2h = hy.numel() * hy.element_size()
    for i in range(3):
        dx.copy_(hx[i % S], non_blocking=True)
        dl.copy_(hl[i % S], non_blocking=True)
        nslm.nslm_moe_stack_decode(arr, LAYERS, E, K_TOP, dl, dx, T, y, ws, wsb)
        hy.copy_(y, non_blocking=True)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for i in range(args.steps):
        dx.copy_(hx[i % S], non_blocking=True)
        dl.copy_(hl[i % S], non_blocking=True)
        nslm.nslm_moe_stack_decode(arr, LAYERS, E, K_TOP, dl, dx, T, y, ws, wsb)
        hy.copy_(y, non_blocking=True)
    f1.record()
    torch.cuda.synchronize()
    e2e_t = slowest_rank_time(f0.elapsed_time(f1) * 1e-3, world, dev)
    e2e = {"value": job_throughput(world, args.steps, T, e2e_t), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h}

    # --- roofline of the dominant kernel: the persistent launch that runs all
    # 45 layers (99% of the step; the routing launch is the rest), from the
    # timed region itself: packed bytes the step reads / measured step time
    step_s = elapsed / args.steps
    ids = torch.empty(T, K_TOP, dtype=torch.int32, device=dev)
    wts = torch.empty(T, K_TOP, device=dev)
    per_expert = layer_packed_bytes_per_token() / K_TOP
    step_bytes = 0.0
    for lg in logits:  # distinct experts per layer, averaged over the cycled inputs
        for l in range(LAYERS):
            step_bytes += len(set(lg[l].topk(K_TOP, dim=-1).indices.reshape(-1).tolist())) * per_expert
    step_bytes /= len(logits)
    achieved = step_bytes / step_s / 1e9
    traffic = None
    warp_instr = None
    rec = layer_record()
    if T == 1 and rec["matches"]:  # the counters hold only for the kernel source they were taken on
        if rec["dram_bytes_per_layer_call"] is not None:  # one layer's DRAM bytes, x the launch's 45 layers
            traffic = rec["dram_bytes_per_layer_call"] * LAYERS
        warp_instr = rec["warp_instructions_per_layer_call"]  # one layer's warp instructions (issue view)
    # one layer through nslm_moe_seed_ffn (routing plan + the persistent
    # kernel for one layer), for context: per-call overheads included
    nslm.nslm_moe_route_topk(logits[0][0], T, E, K_TOP, ids, wts)
    fsb = nslm.nslm_workspace_bytes(nslm.NSLM_OP_MOE_FFN, T, E, HIDDEN, INTER, K_TOP)
    fws = torch.empty(fsb, dtype=torch.uint8, device=dev)
    st = [(nslm.matrix(L.gate), nslm.matrix(L.up), nslm.matrix(L.down)) for L in layers]
    nreps = 4 * LAYERS
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        for i in range(nreps):
            nslm.nslm_moe_seed_ffn(*st[i % LAYERS], E, xs[0], ids, wts, T, K_TOP, y, fws, fsb)
    g.replay()
    torch.cuda.synchronize()
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record()
    g.replay()
    r1.record()
    torch.cuda.synchronize()
    layer_s = r0.elapsed_time(r1) * 1e-3 / nreps
    one_layer = {"workload": "one MoE layer decode: 100 experts, 2048/1408, P=4, top-8, one token "
                             "(routing plan + the persistent kernel for one layer, per call)",
                 "us": round(layer_s * 1e6, 3), "tokens_per_s": round(1.0 / layer_s, 1),
                 "packed_GB_s": round(layer_packed_bytes_per_token() / layer_s / 1e9, 1),
                 "hbm_frac": round(layer_packed_bytes_per_token() / layer_s / 1e9 / hbm, 4),
                 "weights_per_s": round(K_TOP * 3 * HIDDEN * INTER / layer_s, 1)}
    roofline = {"bound": "hbm",
                "kernel": f"{'stack1_kernel' if T == 1 else 'stackb_kernel'}: one cooperative launch running all "
                          f"{LAYERS} layers (with the routing launch, ~1% of the step)",
                "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "traffic": traffic,
                "frac_of_nominal_8TBs": round(achieved / NOMINAL_HBM_GBS, 4),
                "algorithmic_bytes_per_launch": int(step_bytes), "us_per_launch": round(step_s * 1e6, 3),
                "traffic_note": "one layer's ncu DRAM bytes x the launch's layers",
                "single_layer_call_us": round(layer_s * 1e6, 3),
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback"}
    if warp_instr is not None:
        # the bound in practice: the instruction stream that regenerates the
        # weights.  Achieved lane-instructions per second over the timed
        # launch (one layer's ncu count x its layers) against the issue peak:
        # 4 schedulers x 32 lanes x one instruction per clock per SM at the
        # median SM clock sampled under load
        mhz = clk.summary().get("sm_mhz") or clk.summary().get("sm_max_mhz")
        if mhz:
            lanes_s = warp_instr * 32.0 * LAYERS / step_s
            peak_alu = torch.cuda.get_device_properties(dev).multi_processor_count * 128 * mhz * 1e6
            roofline["alu"] = {"bound": "alu", "unit": "lane-instructions/s", "achieved": round(lanes_s, 1),
                               "peak": round(peak_alu, 1), "frac": round(lanes_s / peak_alu, 4),
                               "warp_instructions_per_layer": warp_instr,
                               "peak_basis": f"SMs x 128 lanes x 1 instruction/clock x {mhz} MHz (median under load)"}
    del g
    torch.cuda.empty_cache()

    batched = None
    if not args.no_batched:
        bf16_peak = None
        pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
        if os.path.exists(pk):
            bf16_peak = float(json.load(open(pk)).get("bf16_tflops", 0.0)) or None
        batched = {"workload": "one batched MoE layer on the tensor-core path: 100 experts, 2048/1408, P=3, top-8",
                   "results": batched_sweep(torch, nslm, synth, dev, hbm, bf16_peak),
                   "note": "4 resident layers rotated in a CUDA graph; packed bytes = experts touched"}

    gemv = None
    if not args.no_gemv:
        gemv = {"metric": GEMV_METRIC, "shapes": gemv_sweep(torch, nslm, synth, dev, hbm, args.gemv_shapes),
                "note": "batch 1, each shape timed over rotating copies (> 4x L2) in a CUDA graph (cold, HBM); "
                        "fields_ready_*: the same chain through nslm_seed_gemv_flags(NSLM_GEMV_FIELDS_READY); "
                        "warm_L2_*: one copy repeated, L2-resident; pct_of_nominal_8TBs: of the nominal 8 TB/s"}

    batch8 = None
    if T == 1 and not args.no_batch8:
        batch8 = stack_batch_leg(torch, nslm, synth, dev, arr, hbm, 8, max(10, args.steps // 4), rank)

    p3c5 = None
    if T == 1 and not args.no_p3c5:
        p3c5 = stack_p3c5_leg(torch, nslm, synth, dev, hbm, max(10, args.steps // 4), rank)

    host_experts = None
    if T == 1 and world == 1 and not args.no_host_experts:  # pins 3.9 GB of host memory per process
        host_experts = host_experts_leg(torch, nslm, synth, dev)

    search = None
    if not args.no_search:
        search = search_leg(torch, nslm, dev, with_cpu=(rank == 0 and not args.no_cpu))

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(elapsed / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded SplitMix64 packed fields, bf16 N(0,1) activations, N(0,1) router logits)",
        "config": workload_config(T, world),
        "graph": "one CUDA graph per step",
        "clocks": clk.summary(),
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "roofline": roofline,
    }
    if gemv is not None:
        line["gemv"] = gemv
    if batched is not None:
        line["batched"] = batched
    line["one_layer_decode"] = one_layer
    if batch8 is not None:
        line["stack_batch8"] = batch8
    if p3c5 is not None:
        line["stack_p3c5"] = p3c5
    if host_experts is not None:
        line["host_experts"] = host_experts
    if search is not None:
        line["seed_search"] = search
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line))
    graphs.clear()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
