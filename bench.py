"""Benchmark of the gated-delta-rule tree-verify hot path on B200.

One step = the whole hot path for one verification step of a DDTree budget-22
draft tree (23 nodes: root + 22 drafts) through a 48-GDN-layer stack
(Qwen3.5/3.6-27B geometry: 48 v-heads over 16 k-heads, d_k = d_v = 128, bf16
q/k/v, f32 g/beta/state): gdn_tree_verify on each of the 48 layers (each with
its own buffers), then one gdn_tree_commit_layers call that commits the
accepted root-to-leaf path on every layer (in place: each layer's state_out
aliases its recurrent state).

Metric: tree-nodes/s -- draft-tree nodes carried through all 48 layers and
committed, per second, summed over ranks (weak scaling: every rank verifies
its own independent sequences; no data-path collective).  Also reported:
node-layers/s and algorithmic HBM GB/s of the verify kernel against the
measured copy bandwidth.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                        [--state-dtype f32|f16] [--batch B] [--budget 22] [--layers 48]
Under torchrun (N > 1) every rank runs a replica; rank 0 prints the line.
"""
from __future__ import annotations

import argparse
import contextlib
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gdn_inputs import (ddtree_like_tree, draft_logprobs, make_device_inputs, make_problem,  # noqa: E402
                        root_path)

METRIC = "GDN tree-verify nodes/s and achieved HBM GB/s (% of B200 peak) at budget 22"
UNIT = "tree-nodes/s"
N_K_HEADS, N_V_HEADS, D = 16, 48, 128
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # the B200 HBM3e figure the target is stated against (context beside the measured peak)


# ----------------------------------------------------------------------------
# Algorithmic bytes (what the method must move, per launch; implementation
# re-reads are not counted)
# ----------------------------------------------------------------------------

def verify_bytes(batch, n_nodes, state_dtype, qkv_bytes=2, hk=N_K_HEADS, hv=N_V_HEADS, d=D):
    """Per verify launch: q, k, v (qkv dtype), g, beta (f32), parent (int32),
    out (f32) and every node's persisted state, plus state_in (f32) once per tree."""
    st = 4 if state_dtype == "f32" else 2
    per_node = (2 * hk * d + hv * d) * qkv_bytes + 2 * hv * 4 + 4 + hv * d * 4 + hv * d * d * st
    return batch * (n_nodes * per_node + hv * d * d * 4)


def commit_bytes(batch, state_dtype, hv=N_V_HEADS, d=D):
    st = 4 if state_dtype == "f32" else 2
    return batch * hv * d * d * (st + 4)


# ----------------------------------------------------------------------------
# Distributed plumbing (one process per GPU; torchrun env)
# ----------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(ws, backend):
    import torch.distributed as dist
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def aggregate(local_ms: float, local_units: float, ws: int, device=None):
    """Max of the ranks' timed-region milliseconds and sum of their units.
    Returns (max_ms, total_units, whole-job units/s)."""
    if ws > 1:
        import torch.distributed as dist
        t = torch.tensor([local_ms], dtype=torch.float64, device=device)
        u = torch.tensor([local_units], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(u, op=dist.ReduceOp.SUM)
        local_ms, local_units = float(t.item()), float(u.item())
    return local_ms, local_units, local_units / (local_ms / 1e3)


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------
# Peaks, clocks, ncu traffic record
# ----------------------------------------------------------------------------

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def bf16_tensor_peak():
    """Measured dense bf16 tensor throughput (TFLOP/s, cuBLAS burst), else the
    fallback of this pool's earlier measurement."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


# Tensor-core work of the chunked chain per (CTA, 64-token chunk): one CTA
# holds 128 state rows; kind::f16 products of M = 128 rows, 2 * M * N * K
# flops each, with operands split into bf16 parts (the issued work) and the
# same products at one part each (the chunked form's own arithmetic).
CHUNK_T, CHUNK_ROWS = 64, 128
CHUNK_FLOPS_ISSUED = 2 * CHUNK_ROWS * (
    2 * 2 * CHUNK_T * 128      # X^T | Y^T = S [K; Q]^T, S in 2 parts
    + 2 * CHUNK_T * 128 // 2   # [K; Q] K^T (M = 2T rows of K and Q, N = T)
    + 6 * CHUNK_T * CHUNK_T    # U^T = P^T Ab^T, 6 part products
    + 3 * 128 * CHUNK_T        # S += (U^T diag(r)) K, 3 parts
    + 3 * CHUNK_T * CHUNK_T)   # U^T M^T, 3 part products
CHUNK_FLOPS_ALGO = 2 * CHUNK_ROWS * (
    2 * CHUNK_T * 128 + 2 * CHUNK_T * 128 // 2 + CHUNK_T * CHUNK_T + 128 * CHUNK_T + CHUNK_T * CHUNK_T)


def chunked_tensor_roofline(t: float, batch: int, n_tokens: int) -> dict:
    """Tensor roofline of one GDN_FLAG_CHUNKED launch over ``batch`` chains of
    ``n_tokens`` (48 v-heads, d = 128) that took ``t`` seconds: the issued
    bf16 flops (bf16 parts included) against the measured dense bf16 peak
    (the burst figure: the launch is timed on its own), and the chunked
    form's own flops beside them."""
    ctas = batch * N_V_HEADS * -(-D // CHUNK_ROWS)
    chunks = -(-n_tokens // CHUNK_T)
    issued = ctas * chunks * CHUNK_FLOPS_ISSUED
    tpeak, tkind = bf16_tensor_peak()
    return {"bound": "tensor", "achieved": issued / t / 1e12, "unit": "TFLOP/s", "peak": tpeak,
            "frac": issued / t / 1e12 / tpeak, "peak_source": tkind + " bf16",
            "algorithmic": ctas * chunks * CHUNK_FLOPS_ALGO / t / 1e12, "issued_gflop": issued / 1e9}


def kernel_source_digest():
    """Digest of the sources the verify kernels are built from (the tree
    builder, chunked chain and commit kernels live in files of their own)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_deltanet_tree_verify_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.startswith("gdn_verify") or name in ("gdn_device.cuh", "gdn_internal.h"):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str, units_per_launch: float):
    """DRAM bytes per launch from the committed ncu record, scaled to this
    launch by units processed; None when absent or taken on other kernel code."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel_key]
    except Exception:
        return None
    if rec.get("source_digest") != kernel_source_digest():
        return None
    return rec["dram_bytes_per_unit"] * units_per_launch


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.05):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = "%08X:%02X:%02X.0" % (int(props.pci_domain_id), int(props.pci_bus_id),
                                        int(props.pci_device_id))
            try:
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
            self.ok = True
        except Exception:
            self.ok = False
        self.period = period_s
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.ok:
            self._t.join()

    def now(self):
        """One SM clock reading (MHz), or None."""
        if not self.ok:
            return None
        try:
            return self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM)
        except Exception:
            return None

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# The workload
# ----------------------------------------------------------------------------

class Stack:
    """Per-layer device buffers of one rank's 48-layer verify + commit step."""

    def __init__(self, *, batch, budget, layers, state_dtype, seed, device):
        import gated_deltanet_tree_verify_b200 as gdn
        self.gdn = gdn
        self.batch, self.n_nodes, self.layers = batch, budget + 1, layers
        self.state_dtype = state_dtype
        tdt = torch.float32 if state_dtype == "f32" else torch.float16
        sd = gdn.GDN_F32 if state_dtype == "f32" else gdn.GDN_F16
        self.host, self.dev = [], []
        first = make_problem(batch=batch, n_nodes=self.n_nodes, n_k_heads=N_K_HEADS, n_v_heads=N_V_HEADS,
                             d_k=D, d_v=D, tree="ddtree", seed=seed, qkv_dtype="bf16", accept="leaf")
        self.parent = first.parent.to(device)
        self.accept_path = first.accept_path.to(device)
        self.accept_len = first.accept_len.to(device)
        self.max_path_len = first.accept_path.shape[1]
        for layer in range(layers):
            prob = first if layer == 0 else make_problem(
                batch=batch, n_nodes=self.n_nodes, n_k_heads=N_K_HEADS, n_v_heads=N_V_HEADS, d_k=D, d_v=D,
                tree="given", parents=first.parent.numpy(), seed=seed * 1000 + layer, qkv_dtype="bf16",
                accept="root")
            self.host.append(prob)
            self.dev.append(dict(
                q=prob.q.to(device), k=prob.k.to(device), v=prob.v.to(device), g=prob.g.to(device),
                beta=prob.beta.to(device), state=prob.state_in.to(device),
                out=torch.empty(batch, self.n_nodes, N_V_HEADS, D, device=device),
                ns=torch.empty(batch, self.n_nodes, N_V_HEADS, D, D, device=device, dtype=tdt)))
        self.scale = first.scale
        self.desc = gdn.make_desc(batch=batch, n_nodes=self.n_nodes, n_k_heads=N_K_HEADS,
                                  n_v_heads=N_V_HEADS, d_k=D, d_v=D, scale=self.scale,
                                  qkv_dtype=gdn.GDN_BF16, state_dtype=sd)
        # Layers after the first: the tree and the layer's recurrent state were
        # written before the preceding kernel (the previous layer's verify)
        # was launched, so they may be read while it still runs.
        self.desc_next = gdn.make_desc(batch=batch, n_nodes=self.n_nodes, n_k_heads=N_K_HEADS,
                                       n_v_heads=N_V_HEADS, d_k=D, d_v=D, scale=self.scale,
                                       qkv_dtype=gdn.GDN_BF16, state_dtype=sd,
                                       flags=gdn.GDN_FLAG_EARLY_TREE)
        # Trees walked with stack slots on large grids (f16 states, f32 trees
        # above 32 nodes): the walk is planned once per step and read by all
        # layers.
        self.plan_bytes = gdn.gdn_tree_plan_bytes(self.desc)
        self.plan = (torch.empty(self.plan_bytes // 4, dtype=torch.int32, device=device)
                     if self.plan_bytes else None)

    def verify_all(self, stream=None):
        g = self.gdn
        if self.plan is not None:
            g.gdn_tree_plan(self.desc, self.parent, self.plan, self.plan_bytes, stream=stream)
        for layer, d in enumerate(self.dev):
            desc = self.desc if layer == 0 else self.desc_next
            if self.plan is not None:
                g.gdn_tree_verify_planned(desc, self.plan, d["q"], d["k"], d["v"], d["g"], d["beta"],
                                          self.parent, d["state"], d["out"], d["ns"], plan_bytes=self.plan_bytes,
                                          stream=stream)
            else:
                g.gdn_tree_verify(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], self.parent, d["state"],
                                  d["out"], d["ns"], stream=stream)

    def commit_all(self, stream=None):
        # one launch commits the accepted path on every layer
        self.gdn.gdn_tree_commit_layers(self.desc, [d["ns"] for d in self.dev], self.parent,
                                        self.accept_path, self.accept_len, self.max_path_len,
                                        [d["state"] for d in self.dev], stream=stream)

    def launches_per_step(self):
        return self.layers + (self.layers + 63) // 64 + (1 if self.plan is not None else 0)


def workload_config(args, ws):
    """The workload's config keys, shared by both arms of the benchmark."""
    n_nodes = args.budget + 1
    step_bytes = (verify_bytes(args.batch, n_nodes, args.state_dtype) + commit_bytes(args.batch, args.state_dtype)) \
        * args.layers
    return {"workload": f"ddtree_budget{args.budget}_{args.layers}layers_b{args.batch}",
            "batch_per_rank": args.batch, "global_batch": args.batch * ws, "budget": args.budget,
            "n_nodes": n_nodes, "layers": args.layers, "n_k_heads": N_K_HEADS, "n_v_heads": N_V_HEADS,
            "d_k": D, "d_v": D, "qkv": "bf16", "state_dtype": args.state_dtype,
            "parallelism": f"replicas{ws}",
            "l2": "inputs larger than L2: each step touches %.2f GB of distinct per-layer buffers"
                  % (step_bytes / 1e9)}


def stage(msg):
    print(f"[bench] {time.strftime('%H:%M:%S')} {msg}", file=sys.stderr, flush=True)


def run_ours(args, ws, rank, local):
    import gated_deltanet_tree_verify_b200 as gdn
    gdn.load_library()  # fails loudly when the CUDA library is missing
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(ws, "nccl")
    stage("building the layer stack")
    stack = Stack(batch=args.batch, budget=args.budget, layers=args.layers, state_dtype=args.state_dtype,
                  seed=args.seed + 7919 * rank, device=device)
    stream = torch.cuda.current_stream(device)

    # CUDA graphs of the 48 verify launches and of the 48 commit launches.
    stage("eager warm-up")
    stack.verify_all()
    stack.commit_all()
    torch.cuda.synchronize()
    s = torch.cuda.Stream(device)
    s.wait_stream(stream)
    with torch.cuda.stream(s):
        for _ in range(2):
            stack.verify_all()
            stack.commit_all()
    stream.wait_stream(s)
    torch.cuda.synchronize()
    stage("capturing graphs")
    gv, gc = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(gv):
        stack.verify_all()
    with torch.cuda.graph(gc):
        stack.commit_all()
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        gv.replay()
        gc.replay()
    torch.cuda.synchronize()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    barrier(ws)
    torch.cuda.synchronize()
    stage("timed region")
    sampler = ClockSampler(local)
    nvtx = torch.cuda.nvtx
    with sampler:
        nvtx.range_push("timed steps")
        for i in range(K):
            ev[i][0].record(stream)
            nvtx.range_push("verify x%d" % args.layers)
            gv.replay()
            nvtx.range_pop()
            ev[i][1].record(stream)
            nvtx.range_push("commit x%d" % args.layers)
            gc.replay()
            nvtx.range_pop()
            ev[i][2].record(stream)
        torch.cuda.synchronize()
        nvtx.range_pop()
    barrier(ws)
    verify_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    commit_ms = sum(e[1].elapsed_time(e[2]) for e in ev)
    total_ms = ev[0][0].elapsed_time(ev[-1][2])
    nodes = args.batch * stack.n_nodes * K
    max_ms, all_nodes, value = aggregate(total_ms, nodes, ws, device)

    # Roofline of the dominant kernel (verify): algorithmic bytes per launch over
    # its average launch duration (graph of back-to-back launches, gaps included).
    vb = verify_bytes(args.batch, stack.n_nodes, args.state_dtype)
    avg_verify_s = verify_ms / 1e3 / (K * args.layers)
    achieved = vb / avg_verify_s / 1e9
    peak, peak_kind = hbm_peak()
    traffic = ncu_traffic(f"gdn_verify_{args.state_dtype}", args.batch * stack.n_nodes)
    cb = commit_bytes(args.batch, args.state_dtype)
    avg_commit_s = commit_ms / 1e3 / (K * args.layers)

    # End to end through the public API with host buffers: per step the
    # step's inputs go host->device from pinned memory, the 48 layers' outputs
    # come back device->host; the recurrent state stays resident on the GPU.
    stage("end-to-end leg")
    torch.cuda.nvtx.range_push("end-to-end leg")
    e2e = run_e2e(stack, args, ws, device, stream)
    torch.cuda.nvtx.range_pop()

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": K, "warmup": args.warmup,
        "ms_per_step": max_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": workload_config(args, ws),
        "timing": "CUDA graphs of 48 verify launches + 1 all-layer commit launch, CUDA events per step",
        "node_layers_per_s": value * args.layers,
        "verify_gbps": achieved,
        "commit_gbps": cb / avg_commit_s / 1e9,
        "verify_us_per_launch": avg_verify_s * 1e6,
        "commit_us_per_layer": avg_commit_s * 1e6,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "gdn_verify_kernel", "peak_source": f"{peak_kind} copy bandwidth",
                     "algorithmic_bytes_per_launch": vb,
                     "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                     "nominal_peak": NOMINAL_HBM_GBS},
        "e2e": e2e,
        "gpu_launches": stack.launches_per_step() * K,
        "clocks": sampler.summary(),
    }
    if not args.no_target:
        # every rank runs the same points (replicas); rank 0 reports its own
        stage("target points")
        torch.cuda.nvtx.range_push("target points")
        result["target"] = run_target(args, device, stream, local)
        torch.cuda.nvtx.range_pop()
    if not args.no_chunked:
        # the chunked tensor-core chain on the long-chain workload; a failure
        # here is reported in its key and does not cost the line
        stage("chunked chain point")
        torch.cuda.nvtx.range_push("chunked chain")
        try:
            result["chunked_chain"] = run_chunked_point(local)
        except Exception as exc:  # noqa: BLE001
            result["chunked_chain"] = {"error": f"{type(exc).__name__}: {exc}"}
        torch.cuda.nvtx.range_pop()
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        stage("cpu baseline (oracle)")
        result["cpu_baseline"] = cpu_baseline(args, stack)
    if ws > 1:
        gv.reset()
        gc.reset()
        dist.destroy_process_group()
    return result if rank == 0 else None


# Points of the batched-tree target (>= 70 % of the HBM roofline at budget
# >= 22 with batch >= 8, for f32 and f16 persisted states): (budget, batch,
# persisted state dtype).
TARGET_POINTS = ((22, 8, "f32"), (22, 8, "f16"), (32, 8, "f16"), (64, 8, "f16"), (128, 8, "f16"),
                 (64, 32, "f16"), (128, 32, "f16"))
TARGET_SET_BYTES = 24 << 30  # device memory for one point's distinct layer buffers


def _target_point(budget, batch, state_dtype, *, layers, device, stream, local, seed, min_timed_s=0.25):
    """One target point: the step's 48 verify launches in one CUDA graph (the
    tree planned once per step, as in the headline step), each launch on its
    own layer buffers; layers cycle through as many distinct buffer sets as
    fit in TARGET_SET_BYTES (every set is several times the L2), then one
    all-layer commit launch over the distinct sets.  Timed with CUDA events
    over graph replays, with the SM clock sampled meanwhile."""
    import gated_deltanet_tree_verify_b200 as gdn
    n = budget + 1
    tdt = torch.float32 if state_dtype == "f32" else torch.float16
    sd = gdn.GDN_F32 if state_dtype == "f32" else gdn.GDN_F16
    vb = verify_bytes(batch, n, state_dtype)
    cb = commit_bytes(batch, state_dtype)
    per_set = vb + 2 * batch * N_V_HEADS * D * D * 4
    n_sets = max(2, min(layers, TARGET_SET_BYTES // per_set))
    parent = np.stack([ddtree_like_tree(budget, torch.Generator().manual_seed(seed + b)) for b in range(batch)])
    sets = []
    for l in range(n_sets):
        d = make_device_inputs(parent=parent, n_k_heads=N_K_HEADS, n_v_heads=N_V_HEADS, d_k=D, d_v=D,
                               seed=seed * 1000 + l, device=device)
        d["out"] = torch.empty(batch, n, N_V_HEADS, D, device=device)
        d["ns"] = torch.empty(batch, n, N_V_HEADS, D, D, device=device, dtype=tdt)
        sets.append(d)
    par = sets[0]["parent"]
    scale = D ** -0.5
    desc = gdn.make_desc(batch=batch, n_nodes=n, n_k_heads=N_K_HEADS, n_v_heads=N_V_HEADS, d_k=D, d_v=D,
                         scale=scale, qkv_dtype=gdn.GDN_BF16, state_dtype=sd)
    desc_next = gdn.make_desc(batch=batch, n_nodes=n, n_k_heads=N_K_HEADS, n_v_heads=N_V_HEADS, d_k=D, d_v=D,
                              scale=scale, qkv_dtype=gdn.GDN_BF16, state_dtype=sd, flags=gdn.GDN_FLAG_EARLY_TREE)
    plan_bytes = gdn.gdn_tree_plan_bytes(desc)
    plan = torch.empty(max(plan_bytes, 16) // 4, dtype=torch.int32, device=device) if plan_bytes else None
    # accept the path to the last node taken (a leaf of a best-first tree)
    paths = [root_path(parent[b], n - 1) for b in range(batch)]
    max_len = max(len(pt) for pt in paths)
    path = torch.tensor([pt + [-1] * (max_len - len(pt)) for pt in paths], dtype=torch.int32, device=device)
    plen = torch.tensor([len(pt) for pt in paths], dtype=torch.int32, device=device)

    def verify_step():
        if plan is not None:
            gdn.gdn_tree_plan(desc, par, plan, plan_bytes)
        for l in range(layers):
            d = sets[l % n_sets]
            dd = desc if l == 0 else desc_next
            if plan is not None:
                gdn.gdn_tree_verify_planned(dd, plan, d["q"], d["k"], d["v"], d["g"], d["beta"], par,
                                            d["state_in"], d["out"], d["ns"], plan_bytes=plan_bytes)
            else:
                gdn.gdn_tree_verify(dd, d["q"], d["k"], d["v"], d["g"], d["beta"], par, d["state_in"],
                                    d["out"], d["ns"])

    # the commit writes a separate state_out per set (the headline commits in
    # place; here the inputs must stay for the next replay)
    outs = [torch.empty(batch, N_V_HEADS, D, D, device=device) for _ in range(n_sets)]

    def commit_step():
        gdn.gdn_tree_commit_layers(desc, [d["ns"] for d in sets], par, path, plen, max_len, outs)

    side = torch.cuda.Stream(device)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        verify_step()
        commit_step()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    gv, gc = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(gv):
        verify_step()
    with torch.cuda.graph(gc):
        commit_step()
    for _ in range(3):
        gv.replay()
        gc.replay()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    gv.replay()
    torch.cuda.synchronize()
    reps = max(3, min(200, int(min_timed_s / max(time.perf_counter() - t0, 1e-6))))
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    sampler = ClockSampler(local, period_s=0.01)
    with sampler:
        e[0].record(stream)
        for _ in range(reps):
            gv.replay()
        e[1].record(stream)
        for _ in range(reps):
            gc.replay()
        e[2].record(stream)
        torch.cuda.synchronize()
    verify_s = e[0].elapsed_time(e[1]) / 1e3 / (reps * layers)
    commit_s = e[1].elapsed_time(e[2]) / 1e3 / (reps * n_sets)
    peak, peak_kind = hbm_peak()
    achieved = vb / verify_s / 1e9
    step_gbps = (vb + cb) / (verify_s + commit_s) / 1e9
    point = {"budget": budget, "batch": batch, "n_nodes": n, "state_dtype": state_dtype, "layers": layers,
             "distinct_layer_buffers": n_sets, "planned": plan is not None,
             "verify_us_per_launch": verify_s * 1e6, "commit_us_per_layer": commit_s * 1e6,
             "algorithmic_bytes_per_launch": vb, "achieved_gbps": achieved, "peak_gbps": peak,
             "frac": achieved / peak, "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
             "step_frac": step_gbps / peak, "node_layers_per_s": batch * n / verify_s,
             "reps": reps, "clocks": sampler.summary()}
    del gv, gc
    sets.clear()
    outs.clear()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return point


CHUNKED_POINT = dict(batch=8, n_tokens=4096, reps=40)


def run_chunked_point(local: int) -> dict:
    """The long-chain workload (8 chains of 4096 tokens, 48 v-heads / 16
    k-heads, d = 128, bf16 q/k/v, a = exp(g) in [0.5, 1], last-only f32
    state) through GDN_FLAG_CHUNKED: the mean time of one launch over graph
    replays on two distinct buffer sets (each larger than L2), with its
    tensor roofline and its own clock record."""
    import gated_deltanet_tree_verify_b200 as gdn
    batch, n, reps = CHUNKED_POINT["batch"], CHUNKED_POINT["n_tokens"], CHUNKED_POINT["reps"]
    flags = gdn.GDN_FLAG_CHAIN | gdn.GDN_FLAG_PERSIST_LAST | gdn.GDN_FLAG_CHUNKED
    sampler = ClockSampler(local, period_s=0.01)
    t, R = _verify_point(batch=batch, n_nodes=n, tree="chain", state_dtype="f32", flags=flags, gate="uniform_a",
                         reps=reps, min_bytes=0, sampler=sampler)
    return {"workload": f"long_chain{n}_b{batch}_persist_last_f32", "flags": "GDN_FLAG_CHUNKED",
            "batch": batch, "tokens_per_chain": n, "ms_per_launch": t * 1e3, "tokens_per_s": batch * n / t,
            "buffer_sets": R, "reps": reps, "roofline": chunked_tensor_roofline(t, batch, n),
            "clocks": sampler.summary(),
            "timing": "CUDA graph of one launch per buffer set, replayed back to back; CUDA events around "
                      "the replays"}


def run_target(args, device, stream, local):
    """The batched-tree target points (TARGET_POINTS), each a 48-layer step
    of verify launches timed on its own; see _target_point."""
    peak, peak_kind = hbm_peak()
    points = []
    for budget, batch, sd in TARGET_POINTS:
        torch.cuda.nvtx.range_push(f"target budget {budget} batch {batch} {sd}")
        points.append(_target_point(budget, batch, sd, layers=args.layers, device=device, stream=stream,
                                    local=local, seed=args.seed + 101 * budget + batch))
        torch.cuda.nvtx.range_pop()
    return {"bar": 0.70, "bound": "hbm", "peak": peak, "peak_source": f"{peak_kind} copy bandwidth",
            "nominal_peak": NOMINAL_HBM_GBS, "points": points,
            "met": all(pt["frac"] >= 0.70 for pt in points),
            "timing": "per point: CUDA graph of 48 verify launches (+ tree plan) replayed back to back, CUDA "
                      "events around the replays; distinct buffer sets per layer, each larger than L2"}


def run_e2e(stack, args, ws, device, stream):
    """The step through the public API with host buffers: every step copies
    each layer's q, k, v, g, beta (one packed pinned buffer per layer) and the
    tree to the device, runs the 48 verify launches and the commit, and reads
    every layer's output back.  Layer l + 1's inputs are copied on a copy
    stream while layer l runs, and layer l's output is read back on a third
    stream as soon as it is written; steps do not overlap each other.  The
    step is captured once as a CUDA graph (the library's calls are stream
    operations, so they capture) and replayed per step; every replay copies
    the inputs up and the outputs down again."""
    gdn = stack.gdn
    K = max(3, min(args.steps, args.e2e_steps))
    keys = ("q", "k", "v", "g", "beta")
    host, dev_views = [], []
    for p in stack.host:
        parts = [getattr(p, key).contiguous() for key in keys]
        nbytes = [t.numel() * t.element_size() for t in parts]
        offs = np.cumsum([0] + [(n + 255) // 256 * 256 for n in nbytes])
        hbuf = torch.empty(int(offs[-1]), dtype=torch.uint8).pin_memory()
        dbuf = torch.empty(int(offs[-1]), dtype=torch.uint8, device=device)
        views = {}
        for key, t, o, n in zip(keys, parts, offs[:-1], nbytes):
            hbuf[int(o):int(o) + n].copy_(t.reshape(-1).view(torch.uint8))
            views[key] = dbuf[int(o):int(o) + n].view(t.dtype).view(t.shape)
        host.append((hbuf, dbuf))
        dev_views.append(views)
    host_tree = dict(parent=stack.host[0].parent.pin_memory(), ap=stack.host[0].accept_path.pin_memory(),
                     al=stack.host[0].accept_len.pin_memory())
    outs = [torch.empty(d["out"].shape, dtype=torch.float32).pin_memory() for d in stack.dev]
    h2d = sum(h.numel() for h, _ in host) + sum(t.numel() * t.element_size() for t in host_tree.values())
    d2h = sum(o.numel() * o.element_size() for o in outs)
    copy_s, back_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
    L = len(stack.dev)
    in_ev = [torch.cuda.Event() for _ in range(L)]
    out_ev = [torch.cuda.Event() for _ in range(L)]
    tree_ev = torch.cuda.Event()

    def step(cs, eager):
        """One step on compute stream cs: inputs up on copy_s, launches on cs,
        each layer's output down on back_s once it is written."""
        copy_s.wait_stream(cs)  # the previous step's launches are done with the inputs
        with torch.cuda.stream(copy_s):
            stack.parent.copy_(host_tree["parent"], non_blocking=True)
            stack.accept_path.copy_(host_tree["ap"], non_blocking=True)
            stack.accept_len.copy_(host_tree["al"], non_blocking=True)
            tree_ev.record(copy_s)
            for l, (hbuf, dbuf) in enumerate(host):
                dbuf.copy_(hbuf, non_blocking=True)
                in_ev[l].record(copy_s)
        if eager:
            cs.wait_stream(back_s)  # the previous step's outputs have been read
        cs.wait_event(tree_ev)
        if stack.plan is not None:
            gdn.gdn_tree_plan(stack.desc, stack.parent, stack.plan, stack.plan_bytes, stream=cs)
        for l, (d, v) in enumerate(zip(stack.dev, dev_views)):
            cs.wait_event(in_ev[l])
            desc = stack.desc if l == 0 else stack.desc_next
            if stack.plan is not None:
                gdn.gdn_tree_verify_planned(desc, stack.plan, v["q"], v["k"], v["v"], v["g"], v["beta"],
                                            stack.parent, d["state"], d["out"], d["ns"],
                                            plan_bytes=stack.plan_bytes, stream=cs)
            else:
                gdn.gdn_tree_verify(desc, v["q"], v["k"], v["v"], v["g"], v["beta"], stack.parent, d["state"],
                                    d["out"], d["ns"], stream=cs)
            out_ev[l].record(cs)
        stack.commit_all(stream=cs)
        with torch.cuda.stream(back_s):
            for l, (o, d) in enumerate(zip(outs, stack.dev)):
                back_s.wait_event(out_ev[l])
                o.copy_(d["out"], non_blocking=True)
        cs.wait_stream(back_s)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup // 4)):
            step(stream, True)
        torch.cuda.synchronize()
    # The step as one CUDA graph (its copies are real memcpy nodes, done
    # again on every replay), as a serving loop would run it; eager calls
    # if the capture is refused.
    graph, mode = None, "eager"
    try:
        cap = torch.cuda.Stream(device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            step(cap, False)
        with torch.cuda.stream(stream):
            for _ in range(3):
                graph.replay()
        torch.cuda.synchronize()
        mode = "graph"
    except Exception as e:  # pragma: no cover - depends on the torch build
        stage(f"end-to-end graph capture refused ({type(e).__name__}: {e}); eager calls")
        graph = None
        torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        barrier(ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            if graph is not None:
                graph.replay()
            else:
                step(stream, True)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    ms = e0.elapsed_time(e1)
    max_ms, units, value = aggregate(ms, args.batch * stack.n_nodes * K, ws, device)
    if graph is not None:
        del graph
    api = ("gdn_tree_plan + gdn_tree_verify(_planned) x 48 + gdn_tree_commit_layers with pinned host buffers: "
           "one packed input copy per layer on a copy stream and one output read per layer on a third stream, "
           "overlapped with the launches within a step; ")
    api += ("the step captured once as a CUDA graph and replayed per step (copies included)" if mode == "graph"
            else "eager ctypes calls")
    return {"value": value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": K, "ms_per_step": max_ms / K, "mode": mode, "api": api}


# ----------------------------------------------------------------------------
# CPU oracle legs
# ----------------------------------------------------------------------------

def _oracle_layer_seconds(prob, nthreads, state_dtype, heads=None):
    import oracle
    t0 = time.perf_counter()
    if heads is None:
        oracle.verify_problem(prob, state_dtype=state_dtype, nthreads=nthreads)
    else:
        for h in heads:
            oracle.verify_pair(prob, 0, h, state_dtype=state_dtype)
    return time.perf_counter() - t0


def cpu_baseline(args, stack, budget_s=12.0):
    """The oracle as it stands, on this host's cores, over a bounded sample of
    the same workload: as many of the 48 layers (in order) as fit in about
    ``budget_s`` seconds, at least one.  Scaled to tree-nodes/s through 48 layers."""
    import oracle
    oracle._load()
    nthreads = os.cpu_count() or 1
    _oracle_layer_seconds(stack.host[0], nthreads, args.state_dtype)  # page in
    done, spent = 0, 0.0
    while done < args.layers and (done == 0 or spent < budget_s):
        spent += _oracle_layer_seconds(stack.host[done], nthreads, args.state_dtype)
        done += 1
    per_layer = spent / done
    value = args.batch * stack.n_nodes / (per_layer * args.layers)
    return {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "sample": f"{done} of {args.layers} layers of the same workload (batch {args.batch}, "
                      f"{stack.n_nodes} nodes, 48 heads), {spent:.1f} s, scaled to 48 layers"}


def run_reference(args, ws, rank):
    """The oracle as the reference arm, on this host's cores, on the same
    workload and config as the CUDA arm.  A step is one whole 48-layer step
    (every layer with its own inputs, all 48 v-heads over every core) when
    K + W such steps end within about 150 s; otherwise each step is a bounded
    sample of it (the same number of layers every step, or a slice of v-heads
    of one layer on one thread), timed as it ran, and the throughput is
    scaled to the whole step from the sampled fraction.  ``steps`` and
    ``ms_per_step`` are always what was timed."""
    if rank != 0:
        return None
    import oracle
    oracle._load()
    nthreads = os.cpu_count() or 1
    n_nodes = args.budget + 1
    first = make_problem(batch=args.batch, n_nodes=n_nodes, n_k_heads=N_K_HEADS, n_v_heads=N_V_HEADS, d_k=D,
                         d_v=D, tree="ddtree", seed=args.seed, qkv_dtype="bf16", accept="leaf")
    probs = [first] + [make_problem(batch=args.batch, n_nodes=n_nodes, n_k_heads=N_K_HEADS, n_v_heads=N_V_HEADS,
                                    d_k=D, d_v=D, tree="given", parents=first.parent.numpy(),
                                    seed=args.seed * 1000 + layer, qkv_dtype="bf16", accept="root")
                       for layer in range(1, args.layers)]
    total = args.steps + args.warmup
    budget_s = 150.0
    t_layer = _oracle_layer_seconds(first, nthreads, args.state_dtype)  # also pages the oracle in
    t_layer = min(t_layer, _oracle_layer_seconds(first, nthreads, args.state_dtype))
    if total * t_layer * args.layers <= budget_s:
        layers_per_step, heads, cores = args.layers, None, nthreads
        fraction = 1.0
        sample = (f"whole steps: all {args.layers} layers (own inputs per layer), all 48 v-heads, batch "
                  f"{args.batch}, {n_nodes} nodes, over {nthreads} threads")
    elif total * t_layer <= budget_s:
        layers_per_step = max(1, min(args.layers, int(budget_s / (total * t_layer))))
        heads, cores = None, nthreads
        fraction = layers_per_step / args.layers
        sample = (f"{layers_per_step} of {args.layers} layers per step (all 48 v-heads, batch {args.batch}, "
                  f"{n_nodes} nodes) over {nthreads} threads; throughput scaled to the whole step")
    else:
        t_head = _oracle_layer_seconds(first, 1, args.state_dtype, heads=[0])
        n_heads = max(1, min(N_V_HEADS, int(budget_s / max(total * t_head, 1e-6))))
        layers_per_step, heads, cores = 1, n_heads, 1
        fraction = n_heads / (N_V_HEADS * args.layers)
        sample = (f"{n_heads} of 48 v-heads of one of {args.layers} layers per step (batch {args.batch}, "
                  f"{n_nodes} nodes), single thread; throughput scaled to the whole step")

    def one_step(i):
        t = 0.0
        for j in range(layers_per_step):
            prob = probs[(i * layers_per_step + j) % args.layers]
            if heads is None:
                t += _oracle_layer_seconds(prob, nthreads, args.state_dtype)
            else:
                t += _oracle_layer_seconds(prob, 1, args.state_dtype,
                                           heads=[(i * heads + h) % N_V_HEADS for h in range(heads)])
        return t

    for i in range(args.warmup):
        one_step(i)
    spent = sum(one_step(args.warmup + i) for i in range(args.steps))
    ms_per_step = spent / args.steps * 1e3
    full_step_s = spent / args.steps / fraction
    value = args.batch * n_nodes / full_step_s
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": workload_config(args, ws),
        "timing": "host wall clock (perf_counter) around each oracle call",
        "sample_fraction_of_step": fraction, "ms_per_full_step": full_step_s * 1e3,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------
# Sweep (not the default line): single-layer verify timings over the pages'
# workload shapes, one JSON line per point
# ----------------------------------------------------------------------------

FP32_LANES_PER_SM = 128  # FP32 CUDA-core lanes per SM (B200); 148 SMs


def _verify_point(*, batch, n_nodes, tree, state_dtype, flags=0, gate="softplus", reps=20,
                  min_bytes=512 << 20, seed=11, workspace=False, planned=False, sampler=None):
    """Mean time of one verify launch, over graph replays of R launches on R
    distinct buffer sets (R sized so the sets together exceed min_bytes).
    With ``workspace``, through gdn_tree_verify_ws (one workspace per set);
    with ``planned``, through gdn_tree_verify_planned with each set's plan
    built beforehand (a step builds it once for all its layers).  A
    ``sampler`` (ClockSampler) runs around the timed replays only."""
    import gated_deltanet_tree_verify_b200 as gdn
    persist_last = bool(flags & gdn.GDN_FLAG_PERSIST_LAST)
    tdt = torch.float32 if state_dtype == "f32" else torch.float16
    es = 4 if state_dtype == "f32" else 2
    ns_bytes = batch * (1 if persist_last else n_nodes) * N_V_HEADS * D * D * es
    io_bytes = batch * n_nodes * (45444 - 4) + batch * N_V_HEADS * D * D * 4
    R = max(2, min(16, -(-min_bytes // max(1, ns_bytes + io_bytes))))
    sets = []
    for r in range(R):
        prob = make_problem(batch=batch, n_nodes=n_nodes, n_k_heads=N_K_HEADS, n_v_heads=N_V_HEADS,
                            d_k=D, d_v=D, tree=tree, seed=seed + 1000 * r, qkv_dtype="bf16", gate=gate,
                            accept="root")
        dev = {k: getattr(prob, k).cuda() for k in ("q", "k", "v", "g", "beta", "parent", "state_in")}
        dev["out"] = torch.empty(batch, n_nodes, N_V_HEADS, D, device="cuda")
        dev["ns"] = torch.empty(batch, 1 if persist_last else n_nodes, N_V_HEADS, D, D, device="cuda",
                                dtype=tdt)
        sets.append((prob, dev))
    desc = gdn.make_desc(batch=batch, n_nodes=n_nodes, n_k_heads=N_K_HEADS, n_v_heads=N_V_HEADS, d_k=D,
                         d_v=D, scale=sets[0][0].scale, qkv_dtype=gdn.GDN_BF16,
                         state_dtype=gdn.GDN_F32 if state_dtype == "f32" else gdn.GDN_F16, flags=flags)
    ws_bytes = gdn.gdn_tree_verify_workspace_bytes(desc) if workspace else 0
    for _, d in sets:
        d["ws"] = torch.empty(max(ws_bytes, 16) // 4, device="cuda") if ws_bytes else None
    plan_bytes = gdn.gdn_tree_plan_bytes(desc) if planned else 0
    for _, d in sets:
        d["plan"] = torch.empty(max(plan_bytes, 16) // 4, dtype=torch.int32, device="cuda") if planned else None
        if planned:
            gdn.gdn_tree_plan(desc, d["parent"], d["plan"], plan_bytes)

    def run_all():
        for _, d in sets:
            if d["plan"] is not None:
                gdn.gdn_tree_verify_planned(desc, d["plan"], d["q"], d["k"], d["v"], d["g"], d["beta"],
                                            d["parent"], d["state_in"], d["out"], d["ns"], plan_bytes=plan_bytes)
            elif d["ws"] is not None:
                gdn.gdn_tree_verify_ws(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"],
                                       d["state_in"], d["out"], d["ns"], d["ws"], ws_bytes)
            else:
                gdn.gdn_tree_verify(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"],
                                    d["state_in"], d["out"], d["ns"])

    run_all()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run_all()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_all()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with (sampler if sampler is not None else contextlib.nullcontext()):
        e0.record()
        for _ in range(reps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
    per_launch_s = e0.elapsed_time(e1) / 1e3 / (reps * R)
    del graph
    return per_launch_s, R


def _varlen_point(*, budgets, state_dtype, workspace=False, reps=20, min_bytes=512 << 20, seed=21):
    """Mean time of one gdn_tree_verify_varlen launch over len(budgets)
    DDTree-style trees of those budgets, packed along the node dimension."""
    import gated_deltanet_tree_verify_b200 as gdn
    tdt = torch.float32 if state_dtype == "f32" else torch.float16
    sizes = [b + 1 for b in budgets]
    T, B, Nmax = sum(sizes), len(sizes), max(sizes)
    one = verify_bytes(1, 1, state_dtype) - N_V_HEADS * D * D * 4  # per node
    R = max(2, min(16, -(-min_bytes // (T * one + B * N_V_HEADS * D * D * 4))))
    sets = []
    for r in range(R):
        seqs = [make_problem(batch=1, n_nodes=n, n_k_heads=N_K_HEADS, n_v_heads=N_V_HEADS, d_k=D, d_v=D,
                             tree="ddtree", seed=seed + 1000 * r + i, qkv_dtype="bf16", accept="root")
                for i, n in enumerate(sizes)]
        cat = lambda key: torch.cat([getattr(x, key)[0] for x in seqs]).contiguous().cuda()  # noqa: E731
        d = dict(q=cat("q"), k=cat("k"), v=cat("v"), g=cat("g"), beta=cat("beta"), parent=cat("parent"),
                 state_in=torch.cat([x.state_in for x in seqs]).contiguous().cuda(),
                 cu=torch.tensor([0] + list(np.cumsum(sizes)), dtype=torch.int32).cuda())
        d["out"] = torch.empty(T, N_V_HEADS, D, device="cuda")
        d["ns"] = torch.empty(T, N_V_HEADS, D, D, device="cuda", dtype=tdt)
        sets.append(d)
    desc = gdn.make_desc(batch=B, n_nodes=Nmax, n_k_heads=N_K_HEADS, n_v_heads=N_V_HEADS, d_k=D, d_v=D,
                         scale=float(D) ** -0.5, qkv_dtype=gdn.GDN_BF16,
                         state_dtype=gdn.GDN_F32 if state_dtype == "f32" else gdn.GDN_F16)
    ws_bytes = gdn.gdn_tree_verify_workspace_bytes(desc) if workspace else 0
    for d in sets:
        d["ws"] = torch.empty(max(ws_bytes, 16) // 4, device="cuda") if ws_bytes else None

    def run_all():
        for d in sets:
            gdn.gdn_tree_verify_varlen(desc, d["cu"], T, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"],
                                       d["state_in"], d["out"], d["ns"], d["ws"], ws_bytes)

    run_all()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run_all()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_all()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / (reps * R)
    del graph
    return t, T * one + B * N_V_HEADS * D * D * 4, T


def _build_point(*, batch, budget, max_depth=16, top_k=8, chain_seed=False, reps=50, seed=31):
    """Mean time of one gdn_build_tree launch (graph-replayed back to back),
    and the oracle's time per tree on this host for comparison."""
    import gated_deltanet_tree_verify_b200 as gdn
    from oracle import tree_build as tb
    gen = torch.Generator().manual_seed(seed)
    lp = draft_logprobs(batch, max_depth, top_k, gen)
    lp_d = torch.from_numpy(lp).cuda()
    N = budget + 1
    par = torch.empty(batch, N, dtype=torch.int32, device="cuda")
    dep = torch.empty_like(par)
    rk = torch.empty_like(par)
    sc = torch.empty(batch, N, device="cuda")
    desc = gdn.make_build_desc(batch=batch, max_depth=max_depth, top_k=top_k, budget=budget,
                               flags=gdn.GDN_BUILD_CHAIN_SEED if chain_seed else 0)

    def run_all():
        for _ in range(reps):
            gdn.gdn_build_tree(desc, lp_d, par, node_depth=dep, node_rank=rk, node_score=sc)

    run_all()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            run_all()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / reps
    del graph
    got = par.cpu().numpy()
    want = tb.build_trees(lp, budget, chain_seed)[0]
    t0 = time.perf_counter()
    n_cpu = 0
    while n_cpu < batch and time.perf_counter() - t0 < 2.0:
        tb.build_tree(lp[n_cpu], budget, chain_seed)
        n_cpu += 1
    cpu_per_tree = (time.perf_counter() - t0) / max(1, n_cpu)
    return t, bool((got == want).all()), cpu_per_tree


def _compact_point(*, batch, budget, row_bytes, reps=20, seed=41):
    """Mean time of one gdn_tree_compact launch: the accepted paths' rows of
    DDTree-style trees gathered into path order.  Returns (seconds, bytes
    moved per launch: each accepted row read once and written once)."""
    import gated_deltanet_tree_verify_b200 as gdn
    n = budget + 1
    prob = make_problem(batch=batch, n_nodes=n, n_k_heads=1, n_v_heads=1, d_k=32, d_v=32, tree="ddtree",
                        seed=seed, qkv_dtype="f32", accept="leaf")
    parent = prob.parent.cuda()
    path, length = prob.accept_path.cuda(), prob.accept_len.cuda()
    src = torch.empty(batch * n * row_bytes // 4, device="cuda")
    dst = torch.empty(batch * path.shape[1] * row_bytes // 4, device="cuda")

    def run_all():
        for _ in range(reps):
            gdn.gdn_tree_compact(src, parent, path, length, dst, batch=batch, n_nodes=n, row_bytes=row_bytes)

    run_all()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            run_all()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / reps
    del graph
    return t, 2 * int(prob.accept_len.sum()) * row_bytes


def run_sweep(args):
    import gated_deltanet_tree_verify_b200 as gdn
    gdn.load_library()
    torch.cuda.set_device(0)
    peak, peak_kind = hbm_peak()
    points = []
    for budget in (8, 15, 22, 32, 64, 128):
        for batch in (1, 8, 32):
            for sd in ("f32", "f16"):
                points.append(dict(kind="tree", budget=budget, batch=batch, state_dtype=sd))
                if sd == "f16":
                    points.append(dict(kind="tree", budget=budget, batch=batch, state_dtype=sd, ws=True))
                if sd == "f16" or budget >= 32:
                    points.append(dict(kind="tree", budget=budget, batch=batch, state_dtype=sd, planned=True))
    for sd in ("f32", "f16"):
        points.append(dict(kind="chain16", budget=15, batch=1, state_dtype=sd))
    # varlen: 8 trees of budgets 8..64 in one launch
    for sd, ws in (("f32", False), ("f16", False), ("f16", True)):
        points.append(dict(kind="varlen", budget=0, batch=8, state_dtype=sd, ws=ws))
    points.append(dict(kind="chain4096", budget=4095, batch=8, state_dtype="f32"))
    points.append(dict(kind="chain4096", budget=4095, batch=8, state_dtype="f32", chunked=True))
    for budget in (22, 64, 128, 1023):
        for batch in (1, 8, 64):
            points.append(dict(kind="build", budget=budget, batch=batch))
    # compaction of the accepted paths' outputs (24 KB rows) and f16 states (1.5 MB rows)
    for batch, row in ((1, 24576), (32, 24576), (8, 1572864), (32, 1572864)):
        points.append(dict(kind="compact", budget=64, batch=batch, row_bytes=row))
    if args.sweep_kinds:
        keep = set(args.sweep_kinds.split(","))
        points = [pt for pt in points if pt["kind"] in keep]
    varlen_budgets = [8, 64, 22, 15, 32, 22, 48, 8]
    clocks = ClockSampler(0, period_s=0.01)
    with clocks:
        for pt in points:
            _sweep_point(args, gdn, pt, peak, varlen_budgets, clocks)
    print(json.dumps({"sweep": "clocks", **clocks.summary()}), flush=True)


def _sweep_point(args, gdn, pt, peak, varlen_budgets, clocks):
    """Times one sweep point and prints its JSON line (with the SM clock read
    right after the timed region)."""
    n = pt["budget"] + 1
    if pt["kind"] == "build":
        t, ok, cpu = _build_point(batch=pt["batch"], budget=pt["budget"])
        line = {"sweep": "build_tree", "budget": pt["budget"], "batch": pt["batch"], "max_depth": 16, "top_k": 8,
                "build_us": t * 1e6, "trees_per_s": pt["batch"] / t, "ns_per_pop": t * 1e9 / pt["budget"],
                "matches_oracle": ok, "oracle_us_per_tree": cpu * 1e6}
    elif pt["kind"] == "compact":
        t, moved = _compact_point(batch=pt["batch"], budget=pt["budget"], row_bytes=pt["row_bytes"])
        line = {"sweep": "compact", "budget": pt["budget"], "batch": pt["batch"], "row_bytes": pt["row_bytes"],
                "compact_us": t * 1e6, "gbps": moved / t / 1e9, "frac_of_hbm": moved / t / 1e9 / peak}
    elif pt["kind"] == "varlen":
        t, vb, T = _varlen_point(budgets=varlen_budgets, state_dtype=pt["state_dtype"], workspace=pt["ws"])
        line = {"sweep": "varlen", "budgets": varlen_budgets, "state_dtype": pt["state_dtype"],
                "workspace": pt["ws"], "verify_us": t * 1e6, "node_layers_per_s": T / t,
                "gbps": vb / t / 1e9, "frac_of_hbm": vb / t / 1e9 / peak}
    elif pt["kind"] == "chain4096":
        flags = gdn.GDN_FLAG_CHAIN | gdn.GDN_FLAG_PERSIST_LAST
        if pt.get("chunked"):
            flags |= gdn.GDN_FLAG_CHUNKED
        t, R = _verify_point(batch=pt["batch"], n_nodes=n, tree="chain", state_dtype="f32", flags=flags,
                             gate="uniform_a", reps=3, min_bytes=0)
        tokens = pt["batch"] * n
        io = tokens * (45444 - 4) + 2 * pt["batch"] * N_V_HEADS * D * D * 4
        flops = tokens * N_V_HEADS * D * D * 7.0  # dot S k, a S, u k^T, S q: 7 flops per element
        clock = args.sm_mhz * 1e6
        alu_peak = 148 * FP32_LANES_PER_SM * 2 * clock / 1e12
        line = {"sweep": "chain4096_persist_last" + ("_chunked" if pt.get("chunked") else ""),
                "batch": pt["batch"], "tokens": n,
                "state_dtype": "f32", "verify_ms": t * 1e3, "tokens_per_s": tokens / t,
                "roofline": {"bound": "alu", "achieved": flops / t / 1e12, "unit": "TFLOP/s",
                             "peak": alu_peak, "frac": flops / t / 1e12 / alu_peak,
                             "peak_source": f"148 SMs x 128 FP32 lanes x 2 x {args.sm_mhz:.0f} MHz"},
                "hbm_gbps": io / t / 1e9}
        if pt.get("chunked"):
            # the tensor cores do the chain's work: issued bf16 flops against
            # the measured dense bf16 peak, and the algorithmic share beside it
            line["recurrence_tflops_equivalent"] = line.pop("roofline")["achieved"]
            line["roofline"] = chunked_tensor_roofline(t, pt["batch"], n)
    else:
        tree = "ddtree" if pt["kind"] == "tree" else "chain"
        flags = 0 if pt["kind"] == "tree" else gdn.GDN_FLAG_CHAIN
        t, R = _verify_point(batch=pt["batch"], n_nodes=n, tree=tree, state_dtype=pt["state_dtype"],
                             flags=flags, workspace=pt.get("ws", False), planned=pt.get("planned", False))
        vb = verify_bytes(pt["batch"], n, pt["state_dtype"])
        line = {"sweep": pt["kind"], "budget": pt["budget"], "batch": pt["batch"],
                "state_dtype": pt["state_dtype"], "workspace": pt.get("ws", False),
                "planned": pt.get("planned", False), "verify_us": t * 1e6,
                "node_layers_per_s": pt["batch"] * n / t, "gbps": vb / t / 1e9,
                "frac_of_hbm": vb / t / 1e9 / peak, "buffer_sets": R}
    line["sm_mhz_after"] = clocks.now()
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--state-dtype", choices=["f32", "f16"], default="f32")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--budget", type=int, default=22)
    ap.add_argument("--layers", type=int, default=48)
    ap.add_argument("--seed", type=int, default=2)
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-target", action="store_true",
                    help="skip the batched-tree target points (budget 22-128, batch 8 and 32, f32 and f16)")
    ap.add_argument("--no-chunked", action="store_true",
                    help="skip the chunked tensor-core chain point (8 chains x 4096 tokens)")
    ap.add_argument("--sweep", action="store_true",
                    help="single-layer verify timings over budgets, batches, dtypes and the long chain "
                         "(one JSON line per point; not the benchmark line)")
    ap.add_argument("--sweep-kinds", default="",
                    help="comma-separated subset of the sweep's point kinds (tree, chain16, varlen, chain4096, "
                         "build, compact); default all")
    ap.add_argument("--sm-mhz", type=float, default=1965.0,
                    help="SM clock for the sweep's FP32 ALU roofline (default: the B200 maximum)")
    args = ap.parse_args(argv)
    if args.sweep:
        run_sweep(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    ws, rank, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, ws, rank)
    else:
        res = run_ours(args, ws, rank, local)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
