"""Benchmark of the eSCN hot path on one or more B200s (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload gst_8064] [--impl ours|reference]

A step is one pass of the whole hot path over one synthetic cell: neighbour
list + Wigner rows (egnn_build_graph), the workload's message-passing layers
(egnn_layer_forward, each with its own weights) and the Hamiltonian head
(egnn_hamiltonian_blocks).  The metric is edges per second per forward layer:
value = (directed edges x layers) / device time of the whole step, summed over
ranks (each rank runs an independent replica: the path does not shard, so
scaling is weak).  Inputs are resident in HBM when timing starts; every step
streams far more than the 126 MB L2 (the Wigner rows and the blocks alone are
1.2 GB for the 8,064-atom cell), so no explicit flush is added.

``--impl reference`` times the fp64 CPU oracle on this machine's host cores on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def so2_flops_per_edge(w) -> float:
    """Algorithmic work of the SO(2) linear alone per edge (m = 0 block and the (+m, -m)
    pairs, each pair four products of (n_m C) x (n_m 2C)), x2 FLOP."""
    L, C = w.lmax + 1, w.channels
    macs = (L * C) * (L * 2 * C)
    for m in range(1, w.mmax + 1):
        nm = L - m
        macs += 4 * (nm * C) * (nm * 2 * C)
    return 2.0 * macs


def reduce_ranks(dist, dev, x: float, op: str) -> float:
    """Max or sum of a per-rank scalar over all ranks (float64)."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def layer_flops_per_edge(w) -> float:
    """Algorithmic multiply-add work of one layer per edge (radial MLP + SO(2) linear), x2 FLOP."""
    L, C, K = w.lmax + 1, w.channels, w.n_rbf
    macs = K * C + C * (L * 2 * C) + (L * C) * (L * 2 * C)
    for m in range(1, w.mmax + 1):
        nm = L - m
        macs += 4 * (nm * C) * (nm * 2 * C)
    return 2.0 * macs


TRAFFIC_WORKLOAD = "hfo2_3000"   # the layer call whose DRAM counters are committed (scaled by edges)
TRAFFIC_FILE = os.path.join(ROOT, "profiles", f"layer_traffic_{TRAFFIC_WORKLOAD}.json")
TRAFFIC_SOURCES = ["equivariant_gnn_electronic_b200/csrc/so2_fused.cu", "equivariant_gnn_electronic_b200/csrc/so2_tc.cu",
                   "equivariant_gnn_electronic_b200/csrc/so2_tc.cuh", "equivariant_gnn_electronic_b200/csrc/tc_ptx.cuh",
                   "equivariant_gnn_electronic_b200/csrc/api.cu"]
LAYER_KERNELS = ("edge_dst_kernel", "prep_weights", "gate_rotate_kernel", "layer_fused_kernel", "combine_kernel")


def sources_sha1() -> str:
    import hashlib
    h = hashlib.sha1()
    for f in TRAFFIC_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()


def ingest_traffic(csv_path: str, workload: str, edges: int) -> None:
    """Writes the per-kernel DRAM traffic record of one layer call from an ncu CSV (metrics
    dram__bytes_read.sum, dram__bytes_write.sum, gpu__time_duration.sum; one capture of the
    layer call's launches), stamped with the hash of the kernel sources it was taken on."""
    import csv
    rows = list(csv.reader(open(csv_path)))
    hdr = next(i for i, r in enumerate(rows) if "Kernel Name" in r and "Metric Name" in r)
    cols = rows[hdr]
    ki, mi, vi, ui = cols.index("Kernel Name"), cols.index("Metric Name"), cols.index("Metric Value"), \
        cols.index("Metric Unit")
    idi = cols.index("ID")
    launches = {}
    for r in rows[hdr + 1:]:
        if len(r) <= max(ki, mi, vi, ui):
            continue
        name = next((k for k in LAYER_KERNELS if k in r[ki]), None)
        if name is None:
            continue
        v = float(r[vi].replace(",", ""))
        unit = r[ui].lower()
        scale = {"byte": 1.0, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "nsecond": 1e-6, "usecond": 1e-3,
                 "msecond": 1.0, "ns": 1e-6, "us": 1e-3, "ms": 1.0}.get(unit, 1.0)
        launches.setdefault((r[idi], name), {})[r[mi]] = v * scale
    per = {}
    for (_, name), m in launches.items():
        k = per.setdefault(name, {"kernel": name, "launches": 0, "read_gb": 0.0, "write_gb": 0.0, "ms": 0.0})
        k["launches"] += 1
        k["read_gb"] += m.get("dram__bytes_read.sum", 0.0) / 1e9
        k["write_gb"] += m.get("dram__bytes_write.sum", 0.0) / 1e9
        k["ms"] += m.get("gpu__time_duration.sum", 0.0)
    tot = sum(k["read_gb"] + k["write_gb"] for k in per.values())
    rec = {"workload": workload, "edges": edges, "sources": TRAFFIC_SOURCES, "sources_sha1": sources_sha1(),
           "kernels": list(per.values()), "bytes_per_edge": tot * 1e9 / edges,
           "note": "one ncu capture of one layer call; counters from a single pass per launch"}
    json.dump(rec, open(os.path.join(ROOT, "profiles", f"layer_traffic_{workload}.json"), "w"), indent=1)
    print(json.dumps(rec, indent=1))


def measured_traffic(kernel_prefix=None):
    """DRAM bytes per edge of the dominant kernel (or, without a prefix, of the whole layer
    call) from the committed capture, or None if the kernel sources changed since."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, "no capture"
    d = json.load(open(TRAFFIC_FILE))
    if d.get("sources_sha1") != sources_sha1():
        return None, "kernel sources changed since the capture"
    if kernel_prefix is None:
        return d["bytes_per_edge"], f"layer call, from {d['workload']} ({d['edges']} edges)"
    gb = sum(k["read_gb"] + k["write_gb"] for k in d["kernels"] if k["kernel"].startswith(kernel_prefix))
    return gb * 1e9 / d["edges"], f"{kernel_prefix} bytes per edge from {d['workload']} ({d['edges']} edges)"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            if self.uuid and self.uuid not in f[1]:
                continue
            try:
                sm.append(float(f[2]))
                smax = float(f[3])
            except ValueError:
                continue
            for nm, v in zip(names, f[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def oracle_sample_run(w, pos, box, n_emb, W, atoms, graph=None):
    """Oracle layer over the sampled destination atoms (their full incoming segments).
    The oracle's own neighbour list is built first and not timed."""
    from oracle import graph as og
    from oracle import layer as ol
    rp, src, sh = og.neighbour_list(pos, box, w.rcut) if graph is None else graph
    ne = int(sum(rp[a + 1] - rp[a] for a in atoms))
    t0 = time.perf_counter()
    ol.layer_forward(pos, box, rp, src, sh, n_emb, W, lmax=w.lmax, mmax=w.mmax, rcut=w.rcut,
                     n_rbf=w.n_rbf, heads=w.heads, atoms=atoms)
    return ne, time.perf_counter() - t0, (rp, src, sh)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([x.get("num_threads", 1) for x in info] + [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_baseline(w, pos, box, n_emb, W, atoms):
    """The oracle on this host: the same sample on every BLAS thread, then on one thread."""
    from threadpoolctl import threadpool_limits
    ne, t_all, graph = oracle_sample_run(w, pos, box, n_emb, W, atoms)
    with threadpool_limits(limits=1):
        _, t_one, _ = oracle_sample_run(w, pos, box, n_emb, W, atoms, graph)
    return ne, t_all, t_one


def run_reference(args, w):
    """The oracle on this host's cores: each step = the layer over a bounded atom sample."""
    pos, species, box = synth.make_cell(w, 0)
    n_emb = synth.make_embeddings(w, len(pos), 0)
    W = synth.make_layer_weights(w, 0)
    rng = np.random.default_rng(123)
    per_step = max(4, args.ref_atoms // max(1, args.steps + args.warmup))
    times, edges = [], []
    graph = None
    for i in range(args.warmup + args.steps):
        atoms = np.sort(rng.choice(len(pos), per_step, replace=False))
        ne, dt, graph = oracle_sample_run(w, pos, box, n_emb, W, atoms, graph)
        if i >= args.warmup:
            times.append(dt)
            edges.append(ne)
    value = sum(edges) / sum(times)
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": "edges/sec per fwd eSCN layer", "value": value, "unit": "edges/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "atoms": w.n_atoms, "lmax": w.lmax, "mmax": w.mmax, "channels": w.channels,
                   "heads": w.heads, "layers": w.n_layers, "sample_atoms_per_step": per_step},
        "cpu_baseline": {"value": value, "unit": "edges/s", "cores": cores, "kind": "oracle",
                         "sample": f"layer over {per_step} random destination atoms per step (all their incoming "
                                   f"edges), fp64 numpy oracle"},
        "e2e": {"value": value, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="gst_8064")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-atoms", type=int, default=256)
    ap.add_argument("--cpu-atoms", type=int, default=160, help="oracle sample for cpu_baseline (0: skip)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--ingest-traffic", default=None,
                    help="ncu CSV of one layer call: write the DRAM traffic record for the workload and exit")
    ap.add_argument("--edges", type=int, default=0, help="edges of the captured layer call (with --ingest-traffic)")
    args = ap.parse_args()
    w = synth.WORKLOADS[args.workload]
    if args.ingest_traffic:
        ingest_traffic(args.ingest_traffic, w.name, args.edges)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w)
        return

    import torch
    import torch.distributed as dist
    from equivariant_gnn_electronic_b200 import egnn

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    # ---- inputs (seed = rank: independent replicas) ----
    pos_np, spc_np, box = synth.make_cell(w, rank)
    desc = egnn.desc_for(w)
    dt = egnn.torch_dtype(desc)
    n_np = synth.make_embeddings(w, len(pos_np), rank)
    weights = [egnn.pack_weights(synth.make_layer_weights(w, rank, layer=i), desc, device=dev)
               for i in range(w.n_layers)]
    has_head = len(w.shells) > 0
    head_w = egnn.pack_weights(synth.make_head_weights(w, rank), desc, attention=False, device=dev) \
        if has_head else None
    pos = torch.from_numpy(pos_np).to(dev)
    spc = torch.from_numpy(spc_np).to(dev)
    n0 = torch.from_numpy(n_np.astype(np.float32)).to(dt).to(dev).contiguous()
    g = egnn.build_graph(pos, spc, box, w.rcut, w.lmax, w.mmax)
    E = g.n_edges
    ws_graph = torch.empty(egnn.workspace_bytes(egnn.EGNN_WS_BUILD_GRAPH, None, len(pos_np), 0),
                           dtype=torch.uint8, device=dev)
    ws_layer = torch.empty(max(1, egnn.workspace_bytes(egnn.EGNN_WS_LAYER, desc, len(pos_np), E)),
                           dtype=torch.uint8, device=dev)
    ws_head = torch.empty(egnn.workspace_bytes(egnn.EGNN_WS_HAMILTONIAN, desc, len(pos_np), E),
                          dtype=torch.uint8, device=dev)
    bufs = [torch.empty_like(n0), torch.empty_like(n0)]
    blocks = torch.empty(E, w.n_orb, w.n_orb, dtype=torch.float32, device=dev) if has_head else None
    stream = torch.cuda.current_stream(dev)
    ev_layer = []

    def step(record_layers=False):
        egnn.build_graph(pos, spc, box, w.rcut, w.lmax, w.mmax, workspace=ws_graph, graph=g)
        x = n0
        for i in range(w.n_layers):
            y = bufs[i % 2]
            if record_layers:
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
            egnn.layer_forward(g, desc, weights[i], x, y, workspace=ws_layer)
            if record_layers:
                b.record(stream)
                ev_layer.append((a, b))
            x = y
        if has_head:
            egnn.hamiltonian_blocks(g, desc, head_w, w.shells, x, blocks, workspace=ws_head)
        return x

    # Our kernels per step (tensor-core path): graph build 7 (cell_assign, scan, cell_fill,
    # nbr_count, scan, nbr_fill, wigner); per layer edge_dst and prep_weights, then
    # gate_rotate + layer_fused per range of edge tiles, then combine; the head
    # prep_weights, gate_rotate + so2_gemm per range, head_label.
    n_tiles = (E + 127) // 128
    n_ranges = max(1, -(-n_tiles // 4096))
    launches_per_step = 7 + w.n_layers * (3 + 2 * n_ranges) + ((2 + 2 * n_ranges) if has_head else 0)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert g.read_status() == 0, "device status set during warm-up"
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    egnn.profile(True)   # CUDA events around each SO(2) GEMM launch, on its own stream
    t_start.record(stream)
    for _ in range(args.steps):
        step(record_layers=True)
    t_end.record(stream)
    torch.cuda.synchronize()
    egnn.profile(False)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    layer_ms = [a.elapsed_time(b) for a, b in ev_layer]
    gemm_ms, gemm_n, gemm_edges = egnn.profile_read()
    if world > 1:
        total_ms = reduce_ranks(dist, dev, total_ms, "max")
        edges_all = reduce_ranks(dist, dev, float(E), "sum")
    else:
        edges_all = float(E)
    value = edges_all * w.n_layers * args.steps / (total_ms / 1e3)

    # ---- roofline of the dominant kernel: the fused layer kernel (tcgen05) ----
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    peak_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    layer_avg_s = (sum(layer_ms) / len(layer_ms)) / 1e3
    layer_flops = layer_flops_per_edge(w) * E
    layer_tf = layer_flops / layer_avg_s / 1e12
    per_edge_traffic, traffic_note = measured_traffic("layer_fused")
    layer_traffic, layer_traffic_note = measured_traffic(None)
    per_launch_edges = gemm_edges / gemm_n if gemm_n else float(E)
    gemm_flops = so2_flops_per_edge(w) * per_launch_edges
    gemm_avg_s = gemm_ms / gemm_n / 1e3 if gemm_n else layer_avg_s
    achieved = gemm_flops / gemm_avg_s / 1e12
    roofline = {"bound": "tensor",
                "kernel": "layer_fused_kernel (SO(2) linear on tcgen05 with the attention logits, "
                          "per-atom softmax, rotate-back and aggregation in its epilogue)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "frac_of_burst": achieved / peak_burst,
                "traffic": None if per_edge_traffic is None else per_edge_traffic * per_launch_edges,
                "traffic_note": traffic_note,
                "peak_source": f"bf16_tflops_sustained ({peak_src}); burst {peak_burst}",
                "flops_per_launch": gemm_flops, "flops_counted": "SO(2) blocks only, 8.19 MFLOP per edge at lmax 4",
                "launch_ms": 1e3 * gemm_avg_s, "launches": gemm_n, "edges_per_launch": per_launch_edges,
                "timing": "CUDA events recorded by the library around each launch, on its stream, "
                          "inside the timed region",
                "messages_in_hbm": False}
    roofline["layer_call"] = {"kernels": "edge_dst, prep_weights, (gate_rotate, layer_fused) per edge-tile "
                                         "range, combine",
                              "ms": 1e3 * layer_avg_s, "tflops": layer_tf, "frac": layer_tf / peak,
                              "frac_of_burst": layer_tf / peak_burst,
                              "flops_per_call": layer_flops, "flops_counted": "radial MLP + SO(2), 8.528 MFLOP/edge",
                              "edges_per_s": E / layer_avg_s,
                              "traffic": None if layer_traffic is None else layer_traffic * E,
                              "traffic_note": layer_traffic_note}

    # ---- Label <-> Matrix and Hamiltonian assembly of the step's blocks (timed apart) ----
    label_rows = None
    if has_head and rank == 0:
        def timed(fn, reps=5):
            fn()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / reps
        onsite = torch.zeros(len(pos_np), w.n_orb, w.n_orb, dtype=torch.float32, device=dev)
        all_blocks = torch.cat([onsite, blocks])      # on-site and edge blocks of the cell
        labels = egnn.blocks_to_labels(all_blocks, w.shells)
        t_m2l = timed(lambda: egnn.blocks_to_labels(all_blocks, w.shells))
        t_l2m = timed(lambda: egnn.labels_to_blocks(labels, w.shells))
        t_asm = timed(lambda: egnn.assemble_hamiltonian(g, onsite, blocks))
        nb = all_blocks.shape[0]
        label_rows = {
            "template_orbitals": w.n_orb, "blocks": nb, "labels_per_block": egnn.label_count(w.shells),
            "matrix_to_label_ms": t_m2l, "matrix_to_label_atoms_per_s": len(pos_np) / (t_m2l / 1e3),
            "label_to_matrix_ms": t_l2m, "h_assembly_ms": t_asm,
            "h_orbitals": len(pos_np) * w.n_orb,
            "bytes_per_conversion": nb * (w.n_orb * w.n_orb + egnn.label_count(w.shells)) * 4,
            "note": "one structure's on-site + edge blocks per conversion; the pages quote 7.3e5-1.2e6 "
                    "atoms/s Matrix->Label on one GH200 (context, other hardware)"}

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        pos_h = torch.from_numpy(pos_np).pin_memory()
        spc_h = torch.from_numpy(spc_np).pin_memory()
        n_h = n0.cpu().pin_memory()
        out_h = torch.empty(blocks.shape if has_head else n0.shape, dtype=blocks.dtype if has_head else dt).pin_memory()
        h2d = pos_h.numel() * 8 + spc_h.numel() * 4 + n_h.numel() * n_h.element_size()
        d2h = out_h.numel() * out_h.element_size()
        e2e_steps = max(2, min(args.steps, 5))
        for i in range(e2e_steps + 1):
            if i == 1:
                torch.cuda.synchronize()
                if world > 1:
                    dist.barrier()
                t0 = time.perf_counter()
            pos.copy_(pos_h, non_blocking=True)
            spc.copy_(spc_h, non_blocking=True)
            n0.copy_(n_h, non_blocking=True)
            x = step()
            out_h.copy_(blocks if has_head else x, non_blocking=True)
            torch.cuda.synchronize()
        t_e2e = time.perf_counter() - t0
        if world > 1:
            t_e2e = reduce_ranks(dist, dev, t_e2e, "max")
        e2e = {"value": edges_all * w.n_layers * e2e_steps / t_e2e, "unit": "edges/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "note": "pinned host inputs (positions, species, embeddings) -> full step -> blocks to host; "
                       "weights resident"}

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only) ----
    cpu = None
    if rank == 0 and world == 1 and args.cpu_atoms > 0:
        atoms = np.sort(np.random.default_rng(7).choice(len(pos_np), args.cpu_atoms, replace=False))
        ne, t_all, t_one = oracle_baseline(w, pos_np, box, n_np, synth.make_layer_weights(w, 0), atoms)
        cpu = {"value": ne / t_all, "unit": "edges/s", "cores": blas_threads(), "kind": "oracle",
               "nproc": os.cpu_count(),
               "single_thread": {"value": ne / t_one, "unit": "edges/s", "cores": 1},
               "sample": f"one layer over {len(atoms)} random destination atoms ({ne} edges), fp64 numpy oracle, "
                         f"timed on all BLAS threads and on one"}

    if rank == 0:
        line = {
            "metric": "edges/sec per fwd eSCN layer", "value": value, "unit": "edges/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic",
            "config": {"workload": w.name, "atoms": w.n_atoms, "edges": E, "layers": w.n_layers,
                       "lmax": w.lmax, "mmax": w.mmax, "channels": w.channels, "heads": w.heads,
                       "n_rbf": w.n_rbf, "head_orbitals": w.n_orb,
                       "step": "build_graph + layers + hamiltonian head",
                       "l2": "inputs larger than L2 (per step >1 GB of Wigner rows and blocks)",
                       "parallelism": f"replicas x{world}"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "label_matrix": label_rows,
            "gpu_launches": launches_per_step * args.steps, "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
