#!/usr/bin/env python
"""Benchmark of the fused equivariant edge tensor-product convolution on B200.

One step = one pass of the whole hot path over one batch of synthetic input: neighbour list and
canonical CSR from the atom positions, fused forward convolution, fused backward (VJP to node
features and edge vectors) and force assembly. Workload: the 1000-atom periodic diamond cell
(5x5x5 conventional cells, a = 3.567 A, jitter N(0, 0.05 A), r_cut 5 A, 64x0e+64x1o+64x2e,
SH lmax 2, 8 Bessel functions), synthetic seeded inputs, fp32 throughout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {etp,reference}] [--workload NAME]

Multi-GPU (torchrun, one rank per GPU): independent replicas (the path does not shard on one
GPU's workload; weak scaling), no data-path collective; the timed region is the max over ranks.
The reference arm (--impl reference) times the float64 CPU oracle on a bounded sample of the
same workload (rank 0 only).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "edges/sec for TP conv fwd and fwd+bwd (fp32), % of HBM/FP32 roofline"
SM_COUNT = 148
FP32_LANES_PER_SM = 128
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_WARMUP = 20
KERNEL_REPS = 200


def set_kernel_timing(reps, warmup):
    """Calls per kernel timing: the defaults above for measurements; a profiler run of the same
    command lowers them so that every launch can be captured."""
    global KERNEL_REPS, KERNEL_WARMUP
    KERNEL_REPS = max(1, int(reps))
    KERNEL_WARMUP = max(0, int(warmup))
# the other workloads (besides the diamond1k headline) and their oracle sample sizes (receivers),
# chosen so that each float64 sample takes a few seconds on one host core
OTHER_WORKLOADS = ("tiny", "sweep1", "sweep2", "sweep3", "diamond8k", "melt32k")
ORACLE_SAMPLE = {"tiny": 32, "sweep1": 256, "sweep2": 48, "sweep3": 12, "diamond8k": 8, "melt32k": 16}


# ---------------------------------------------------------------- peaks and counts

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": 1965.0}, "fallback"


def fp32_peak_tflops(sm_mhz):
    """Plain FP32 ALU peak: 148 SMs x 128 FP32 lanes x 2 flop (FMA) x SM clock."""
    return SM_COUNT * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12


def launches_per_step(info, n_nodes, min_image=True):
    """Kernels of this library launched by one step (checked against the ncu launch list).

    neighbour list: chunk counts, scan init, scan, row pointers, emit, then for orthorhombic cells
    wider than 2 r_cut (every workload here) the reverse-edge transpose, otherwise iota, radix
    histogram, radix exclusive sum, one onesweep pass per 8 key bits and the row pointers;
    forward: weight split, fused forward; backward: weight split, edge receivers, fused backward,
    unit sum (more than one 16-channel unit); forces: one.
    """
    key_bits = max(1, int(n_nodes).bit_length())
    graph = 6 if min_image else 5 + 4 + (key_bits + 7) // 8
    units = (info["channels"] + 15) // 16
    return graph + 2 + 3 + (1 if units > 1 else 0) + 1


def algorithmic_counts(info, n_nodes, n_edges):
    """Per-launch algorithmic flops / bytes of the plain definition (see the design notes).

    forward  FP32: 2 (nnz + sum_p(2 l3 + 1)) C per edge   (CG contraction with c = C Y, then w s)
    backward FP32: 2 (3 nnz + 2 sum_p(2 l3 + 1)) C per edge (grad_x, grad_w, grad_Y contractions)
    radial projection (tensor-core class work, not counted as FP32): 2 n_basis P C per edge
    (forward), twice that in the backward.
    Compulsory HBM bytes: node rows read/written once, edge arrays once.
    """
    c, nnz, s3 = info["channels"], info["cg_nnz"], info["sum_2l3p1"]
    dim = info["dim_in"]
    fwd_flop = 2.0 * (nnz + s3) * c * n_edges
    bwd_flop = 2.0 * (3 * nnz + 2 * s3) * c * n_edges
    radial = 2.0 * info["n_basis"] * info["n_paths"] * c * n_edges
    fwd_bytes = 4.0 * (2 * n_nodes * dim + 4 * n_edges + n_nodes + 1)
    bwd_bytes = 4.0 * (3 * n_nodes * dim + 4 * n_edges + 3 * n_edges + 2 * (n_nodes + 1) + n_edges)
    # weight gradient (etp_backward_weights): the per-path factor costs what the forward contraction
    # does, and the edge reduction sum_e R_b gw runs on the FP32 pipe too (2 n_basis P C per edge)
    dw_flop = fwd_flop + radial
    dw_bytes = 4.0 * (2 * n_nodes * dim + 4 * n_edges + n_edges + n_nodes + 1)
    return dict(fwd_flop=fwd_flop, bwd_flop=bwd_flop, dw_flop=dw_flop, fwd_radial_flop=radial,
                bwd_radial_flop=2 * radial, fwd_bytes=fwd_bytes, bwd_bytes=bwd_bytes, dw_bytes=dw_bytes)


# ---------------------------------------------------------------- recorded DRAM traffic

CSRC = os.path.join(ROOT, "equivariant_mlip_tensor_edge_b200", "csrc")
FWD_KERNEL = "k_fwd_cx"     # the default forward for l_max <= 2 and 4 <= C <= 64 (C % 4 == 0)
DW_KERNEL = "k_dw_pair"     # the weight gradient for l_max <= 2 (k_dw serves l_max 3)
KERNEL_SOURCES = {
    "k_fwd_cx": ["etp_fwd_cx.cu", "etp_tc_common.h", "etp_device.h", "generated/etp_paths.h"],
    "k_fwd_tc": ["etp_fwd_tc.cu", "etp_tc_common.h", "etp_device.h", "generated/etp_paths.h"],
    "k_bwd_tc": ["etp_bwd_tc.cu", "etp_tc_common.h", "etp_device.h", "generated/etp_paths.h"],
    "k_dw": ["etp_dw.cu", "etp_device.h", "generated/etp_paths.h"],
    "k_dw_pair": ["etp_dw.cu", "etp_device.h", "generated/etp_paths.h"],
    "k_node_ladder": ["etp_product.cu", "etp_device.h", "generated/etp_paths.h"],
    "k_gen_fwd": ["etp_general.cu", "etp_device.h", "generated/etp_paths.h"],
    "k_gen_fwd_tc": ["etp_general_tc.cu", "etp_tc_common.h", "etp_device.h", "generated/etp_paths.h"],
    "k_gen_bwd": ["etp_general.cu", "etp_device.h", "generated/etp_paths.h"],
    "k_gen_dw": ["etp_general.cu", "etp_device.h", "generated/etp_paths.h"],
    "k_ladder_mix": ["etp_ladder_full.cu", "etp_tc_common.h", "etp_device.h", "generated/etp_paths.h"],
}
# dram__bytes_read.sum + dram__bytes_write.sum of one launch, from the ncu captures summarised in
# profiles/<kernel>_<workload>.md, keyed by a hash of the kernel's sources at capture time.
RECORDED_TRAFFIC = {
    ("k_fwd_cx", "diamond1k"): (3838720 + 0, "40b5d99bc09974bb"),
    ("k_bwd_tc", "diamond1k"): (6546944 + 0, "b52ffa427ab48b75"),
    ("k_dw_pair", "diamond1k"): (6418816 + 0, "86c17c159f9a5c2f"),
    ("k_node_ladder", "ladder4096_l2"): (18898432 + 0, "e21b6756156138a7"),
    ("k_gen_fwd_tc", "nequipl_diamond1k"): (4399872 + 0, "ee151666faecb84b"),
    ("k_gen_bwd", "nequipl_diamond1k"): (7565824 + 0, "fcb3a1d2171be5f7"),
    ("k_gen_dw", "nequipl_diamond1k"): (7538176 + 0, "fcb3a1d2171be5f7"),
    ("k_ladder_mix", "ladder_full4096_l2"): (93742976 + 397440, "f4fd8ff8fff3e133"),
}


def source_hash(kernel):
    import hashlib
    m = hashlib.sha1()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), "rb") as fh:
            m.update(fh.read())
    return m.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """Bytes per launch from the recorded capture, or None once the kernel source has changed."""
    rec = RECORDED_TRAFFIC.get((kernel, workload))
    if rec is None or not os.path.isdir(CSRC) or source_hash(kernel) != rec[1]:
        return None
    return rec[0]


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- ranks

def combine_ranks(times_ms, edges, world, device):
    """Whole-job numbers of a multi-rank run: every timing is the maximum over the ranks (the
    slowest replica sets the step time) and the edges are summed (every replica's edges count
    toward the job's throughput). A no-op for one rank."""
    import torch
    t = torch.tensor(list(times_ms), dtype=torch.float64, device=device)
    e = torch.tensor([float(edges)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(e, op=dist.ReduceOp.SUM)
    return t.tolist(), e.item()


# ---------------------------------------------------------------- GPU arm

def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import equivariant_mlip_tensor_edge_b200 as etp
    import workloads

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = workloads.make(args.workload)
    conv = etp.EdgeConv(wl.irreps, wl.lmax, wl.irreps, wl.n_basis, float(wl.r_cut))
    info = conv.info
    pos_h = torch.from_numpy(wl.pos).pin_memory()
    x_h = torch.from_numpy(wl.features()).pin_memory()
    W_h = torch.from_numpy(wl.weights(conv.n_paths)).pin_memory()
    g_h = torch.from_numpy(wl.cotangent()).pin_memory()
    pos, x, W, gout = (t.to(dev) for t in (pos_h, x_h, W_h, g_h))
    n = wl.n_nodes

    g0 = etp.neighbors(pos, float(wl.r_cut), cell=wl.cell, pbc=wl.pbc)
    cap = int(g0.n_edges * 1.25) + 1024
    # persistent buffers (capacity cap) so a step allocates nothing
    bufs = dict(
        row_ptr=torch.empty(n + 1, dtype=torch.int32, device=dev),
        t_row_ptr=torch.empty(n + 1, dtype=torch.int32, device=dev),
        sender=torch.empty(cap, dtype=torch.int32, device=dev),
        edge_vec=torch.empty((cap, 3), dtype=torch.float32, device=dev),
        t_perm=torch.empty(cap, dtype=torch.int32, device=dev),
        gws=torch.empty(etp.graph_workspace_bytes(n, cap), dtype=torch.uint8, device=dev),
        ws=torch.empty(conv.workspace_bytes(n, cap), dtype=torch.uint8, device=dev),
        out=torch.empty((n, info["dim_out"]), dtype=torch.float32, device=dev),
        gx=torch.empty((n, info["dim_in"]), dtype=torch.float32, device=dev),
        gv=torch.empty((cap, 3), dtype=torch.float32, device=dev),
        f=torch.empty((n, 3), dtype=torch.float32, device=dev),
        dw=torch.empty((info["n_basis"], info["n_paths"], info["channels"]), dtype=torch.float32, device=dev),
    )
    lib = etp.load_library()
    import ctypes
    cell_arr = (ctypes.c_double * 9)(*[float(v) for row in wl.cell for v in row]) if wl.cell is not None else None
    pbc_arr = (ctypes.c_int * 3)(*[int(bool(p)) for p in wl.pbc])
    P = etp._ptr
    stream = etp._stream(dev)
    n_edges_c = ctypes.c_int(0)

    def graph_step(pos_d):
        st = lib.etp_neighbors(P(pos_d), n, ctypes.cast(cell_arr, etp._dp) if cell_arr is not None else None,
                               pbc_arr, float(wl.r_cut), cap, ctypes.byref(n_edges_c), P(bufs["row_ptr"]),
                               P(bufs["sender"]), P(bufs["edge_vec"]), None, P(bufs["t_row_ptr"]), P(bufs["t_perm"]),
                               P(bufs["gws"]), bufs["gws"].numel(), stream)
        etp._check(st, "etp_neighbors")
        e = n_edges_c.value
        return etp.Graph(n, e, bufs["row_ptr"], bufs["sender"][:e], bufs["edge_vec"][:e], bufs["t_row_ptr"],
                         bufs["t_perm"][:e])

    def conv_fwd(gr, xx, WW):
        return conv.forward(gr, xx, WW, out=bufs["out"], workspace=bufs["ws"])

    def conv_bwd(gr, xx, WW, gg):
        return conv.backward(gr, xx, WW, gg, grad_x=bufs["gx"], grad_vec=bufs["gv"][:gr.n_edges],
                             workspace=bufs["ws"])

    def step(pos_d, xx, WW, gg):
        gr = graph_step(pos_d)
        conv_fwd(gr, xx, WW)
        conv_bwd(gr, xx, WW, gg)
        etp.forces(gr, bufs["gv"][:gr.n_edges], out=bufs["f"])
        return gr

    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)   # > 126 MB L2

    def timed(fn, k, host_ahead=False):
        """Mean device time of fn over k calls (the step's contract: exactly k timed calls), L2
        flushed before each. host_ahead: a device-side sleep after the flush lets the host enqueue
        fn entirely before the first event, so the time is the kernels' alone, not the host's
        launch latency."""
        return statistics.fmean(event_times(fn, k, host_ahead))

    def event_times(fn, k, host_ahead):
        out = []
        for _ in range(k):
            flush.fill_(1.0)
            if host_ahead:
                torch.cuda._sleep(400_000)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            out.append(a.elapsed_time(b))
        return out

    def kernel_ms(fn):
        """Median device time of one call over KERNEL_REPS calls after KERNEL_WARMUP untimed ones,
        L2 flushed before each call."""
        for _ in range(KERNEL_WARMUP):
            fn()
        return statistics.median(event_times(fn, KERNEL_REPS, True))

    # warm-up
    for _ in range(args.warmup):
        step(pos, x, W, gout)
    torch.cuda.synchronize()
    gr = graph_step(pos)
    torch.cuda.synchronize()

    sampler = ClockSampler(local_rank if os.environ.get("CUDA_VISIBLE_DEVICES") is None else 0)
    if rank == 0:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ms_step = timed(lambda: step(pos, x, W, gout), args.steps)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    # per-kernel timings on the same stream (median of KERNEL_REPS calls after KERNEL_WARMUP)
    ms_fwd = kernel_ms(lambda: conv_fwd(gr, x, W))
    ms_bwd = kernel_ms(lambda: conv_bwd(gr, x, W, gout))
    ms_graph = kernel_ms(lambda: graph_step(pos))
    ms_dw = kernel_ms(lambda: conv.backward_weights(gr, x, gout, grad_W=bufs["dw"], workspace=bufs["ws"]))
    # node-local product ladder: 4096 nodes x 128 channels, correlation order 3, the workload's rank
    lad = dict(n=4096, c=128, nu=3, lmax=wl.lmax)
    gen = torch.Generator().manual_seed(1234)
    lad_dim = (lad["lmax"] + 1) ** 2 * lad["c"]
    lad_A = torch.randn((lad["n"], lad_dim), generator=gen).to(dev)
    lad_W = (torch.randn((lad["nu"] - 1, info["n_paths"], lad["c"]), generator=gen) / info["n_paths"] ** 0.5).to(dev)
    lad_out = torch.empty_like(lad_A)
    for _ in range(3):
        etp.node_ladder(lad_A, lad_W, lad["lmax"], out=lad_out)
    ms_ladder = kernel_ms(lambda: etp.node_ladder(lad_A, lad_W, lad["lmax"], out=lad_out))
    # the full ladder (per-rank path- and channel-mixing matrices on the tensor cores), same size
    lf_W = (torch.randn((lad["nu"] - 1, etp.node_ladder_full_step_floats(lad["lmax"], lad["c"])), generator=gen) /
            (4 * lad["c"]) ** 0.5).to(dev)
    lf_out = torch.empty_like(lad_A)
    lf_ws = torch.empty(etp.load_library().etp_node_ladder_full_workspace_bytes(lad["lmax"], lad["c"], lad["n"]),
                        dtype=torch.uint8, device=dev)
    for _ in range(3):
        etp.node_ladder_full(lad_A, lf_W, lad["lmax"], out=lf_out, workspace=lf_ws)
    ms_ladder_full = kernel_ms(lambda: etp.node_ladder_full(lad_A, lf_W, lad["lmax"], out=lf_out, workspace=lf_ws))
    # general irreps: NequIP-L channel counts on the same graph (table-driven kernels)
    gen_irreps = "128x0e+64x1o+32x2e+32x3o"
    gconv = etp.EdgeConv(gen_irreps, 3, gen_irreps, wl.n_basis, float(wl.r_cut))
    gi = gconv.info
    g_x = torch.randn((n, gi["dim_in"]), generator=gen).to(dev)
    g_W = (torch.randn((gi["n_basis"], gi["weight_numel"] // gi["n_basis"]), generator=gen)
           / gi["n_paths"] ** 0.5).to(dev)
    g_g = torch.randn((n, gi["dim_out"]), generator=gen).to(dev)
    g_ws = torch.empty(max(gconv.workspace_bytes(n, cap), 1), dtype=torch.uint8, device=dev)
    g_out = torch.empty((n, gi["dim_out"]), device=dev)
    g_gx = torch.empty((n, gi["dim_in"]), device=dev)
    g_gv = torch.empty((cap, 3), device=dev)
    gen_fwd = lambda: gconv.forward(gr, g_x, g_W, out=g_out, workspace=g_ws)
    gen_bwd = lambda: gconv.backward(gr, g_x, g_W, g_g, grad_x=g_gx, grad_vec=g_gv[:gr.n_edges], workspace=g_ws)
    for _ in range(3):
        gen_fwd()
        gen_bwd()
    g_dw = torch.empty((gi["n_basis"], gi["weight_numel"] // gi["n_basis"]), device=dev)
    gen_dw = lambda: gconv.backward_weights(gr, g_x, g_g, grad_W=g_dw, workspace=g_ws)
    gen_dw()
    ms_gen_fwd = kernel_ms(gen_fwd)
    ms_gen_bwd = kernel_ms(gen_bwd)
    ms_gen_dw = kernel_ms(gen_dw)
    # every other workload of the benchmark set: forward (and backward) edges/s and roofline
    # fractions, each with its own bounded float64 oracle sample on the host
    others = {}
    if not args.headline_only:
        for name in OTHER_WORKLOADS:
            others[name] = measure_workload(name, dev, kernel_ms, fp32_peak_tflops(measured_peaks()[0].get(
                "sm_max_mhz", 1965.0)), with_oracle=(world == 1 and not args.no_cpu_baseline))
    clocks = sampler.stop() if rank == 0 else None

    # end to end through the public API with host buffers (copies inside the timed region)
    out_h = torch.empty_like(bufs["out"], device="cpu").pin_memory()
    f_h = torch.empty((n, 3), dtype=torch.float32).pin_memory()

    # the copies overlap the compute where the data flow allows: x and W travel (upload stream)
    # while the neighbour list is built from the positions, the cotangent while the forward runs,
    # and the forward output comes back (download stream) while the backward runs
    up_stream = torch.cuda.Stream(device=dev)
    down_stream = torch.cuda.Stream(device=dev)
    ev_xw = torch.cuda.Event()
    ev_g = torch.cuda.Event()
    in_d = [torch.empty_like(t, device=dev) for t in (pos_h, x_h, W_h, g_h)]

    def e2e_step():
        main = torch.cuda.current_stream(dev)
        up_stream.wait_stream(main)                    # the previous step is done with the buffers
        down_stream.wait_stream(main)
        in_d[0].copy_(pos_h, non_blocking=True)
        with torch.cuda.stream(up_stream):
            in_d[1].copy_(x_h, non_blocking=True)
            in_d[2].copy_(W_h, non_blocking=True)
            ev_xw.record(up_stream)
            in_d[3].copy_(g_h, non_blocking=True)
            ev_g.record(up_stream)
        gr_ = graph_step(in_d[0])
        main.wait_event(ev_xw)
        conv_fwd(gr_, in_d[1], in_d[2])
        down_stream.wait_stream(main)
        with torch.cuda.stream(down_stream):
            out_h.copy_(bufs["out"], non_blocking=True)
        main.wait_event(ev_g)
        conv_bwd(gr_, in_d[1], in_d[2], in_d[3])
        etp.forces(gr_, bufs["gv"][:gr_.n_edges], out=bufs["f"])
        f_h.copy_(bufs["f"], non_blocking=True)
        main.wait_stream(down_stream)
        main.wait_stream(up_stream)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    ms_e2e = timed(e2e_step, args.steps)
    h2d = sum(t.numel() * t.element_size() for t in (pos_h, x_h, W_h, g_h))
    d2h = out_h.numel() * 4 + f_h.numel() * 4

    e = gr.n_edges
    (ms_step, ms_e2e, ms_fwd, ms_bwd, ms_graph, ms_dw, ms_ladder, ms_ladder_full, ms_gen_fwd, ms_gen_bwd,
     ms_gen_dw), total_edges = \
        combine_ranks([ms_step, ms_e2e, ms_fwd, ms_bwd, ms_graph, ms_dw, ms_ladder, ms_ladder_full, ms_gen_fwd,
                       ms_gen_bwd, ms_gen_dw],
                      e, world, dev)
    if rank != 0:
        return None

    peaks, peak_kind = measured_peaks()
    sm_max = peaks.get("sm_max_mhz", 1965.0)
    fp32_peak = fp32_peak_tflops(sm_max)
    cnt = algorithmic_counts(info, n, e)
    dominant = "bwd" if ms_bwd >= ms_fwd else "fwd"

    def roof(kind, ms):
        flop = cnt[f"{kind}_flop"]
        ach = flop / (ms * 1e-3) / 1e12
        kernel = {"bwd": "k_bwd_tc", "fwd": FWD_KERNEL, "dw": DW_KERNEL}[kind]
        return {"bound": "alu", "achieved": round(ach, 3), "peak": round(fp32_peak, 2), "unit": "TFLOP/s",
                "frac": round(ach / fp32_peak, 4), "traffic": recorded_traffic(kernel, wl.name),
                "kernel": kernel,
                "timed": {"bwd": "the whole etp_backward call (k_bprep, k_recv_of_edge, k_bwd_tc, k_sum_units)",
                          "fwd": f"the whole etp_forward call (k_cx_prep, {FWD_KERNEL})",
                          "dw": f"the whole etp_backward_weights call (k_recv_of_edge, {DW_KERNEL}, k_dw_sum)"}[kind],
                "peak_source": f"derived: 148 SM x 128 FP32 lanes x 2 x {sm_max:.0f} MHz ({peak_kind} sm_max_mhz)",
                "ms_per_launch": round(ms, 5),
                "hbm_frac_of_" + peak_kind: round(cnt[f"{kind}_bytes"] / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}

    def ladder_roof(ms):
        """The ladder's bound is the slower of its compulsory HBM bytes (A read, out written, W) and
        its FP32 work (3 nnz + 2 sum_p(2 l3 + 1) flop per node, channel and step)."""
        steps = lad["nu"] - 1
        flop = float(3 * info["cg_nnz"] + 2 * info["sum_2l3p1"]) * lad["c"] * lad["n"] * steps
        byts = 4.0 * (2 * lad["n"] * lad_dim + steps * info["n_paths"] * lad["c"])
        t_alu = flop / (fp32_peak * 1e12)
        t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
        if t_hbm >= t_alu:
            ach, peak, unit, bound = byts / (ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s", "hbm"
        else:
            ach, peak, unit, bound = flop / (ms * 1e-3) / 1e12, fp32_peak, "TFLOP/s", "alu"
        return {"workload": f"{lad['n']} nodes x {lad['c']} channels, lmax {lad['lmax']}, order {lad['nu']}",
                "kernel": "k_node_ladder", "ms_per_launch": round(ms, 5), "bound": bound,
                "achieved": round(ach, 3), "peak": round(peak, 2), "unit": unit, "frac": round(ach / peak, 4),
                "peak_source": peak_kind, "traffic": recorded_traffic("k_node_ladder", f"ladder4096_l{lad['lmax']}"),
                "alu_frac": round(flop / (ms * 1e-3) / 1e12 / fp32_peak, 4),
                "hbm_frac_of_" + peak_kind: round(byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}

    def ladder_full_roof(ms):
        """The full ladder's dominant work is the mixing GEMM, 2 K C flop per (node, component) and
        step (K = paths of the component's rank x C); bound: the tensor cores at the TF32 rate (the
        measured bf16 rate x the nominal TF32/bf16 ratio 1.1/2.25). The mixing runs as three TF32
        products (hi*hi + hi*lo + lo*hi) for fp32 accuracy, so the ceiling of this kernel is a third
        of that rate; fp32_frac compares with the FP32 CUDA-core peak an fp32 GEMM would otherwise
        run on."""
        L, c = lad["lmax"], lad["c"]
        paths = [(a, b, d) for a in range(L + 1) for b in range(L + 1) for d in range(L + 1)
                 if abs(a - b) <= d <= a + b and (a + b + d) % 2 == 0]
        per_node = sum((2 * d + 1) * sum(1 for p in paths if p[2] == d) * c * c * 2 for d in range(L + 1))
        flop = float(per_node) * lad["n"] * (lad["nu"] - 1)
        tf32 = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS)) * 1.1 / 2.25
        ach = flop / (ms * 1e-3) / 1e12
        return {"workload": f"{lad['n']} nodes x {c} channels, lmax {L}, order {lad['nu']}, full ladder",
                "kernel": "k_ladder_mix", "ms_per_launch": round(ms, 5), "bound": "tensor",
                "achieved": round(ach, 3), "peak": round(tf32, 2), "unit": "TFLOP/s", "frac": round(ach / tf32, 4),
                "peak_source": f"{peak_kind} bf16 x 1.1/2.25 (TF32)",
                "traffic": recorded_traffic("k_ladder_mix", f"ladder_full4096_l{L}"),
                "fp32_frac": round(ach / fp32_peak, 4), "mixing_gflop": round(flop / 1e9, 3)}

    def general_roof(ms, kind):
        # the weight gradient's per-path factor costs what the forward contraction does, plus the
        # edge reduction sum_e R_b gw (2 n_basis cols flop per edge)
        flop = (float(gi["flop_fwd"]) + 2.0 * gi["weight_numel"]) * e if kind == "dw" else float(gi[f"flop_{kind}"]) * e
        ach = flop / (ms * 1e-3) / 1e12
        # the forward runs the tensor-core general kernel (radial projection on tcgen05)
        kernel = "k_gen_fwd_tc" if kind == "fwd" else f"k_gen_{kind}"
        return {"workload": f"{gen_irreps}, harmonics to l = 3, {wl.name} graph ({e} edges)",
                "kernel": kernel, "ms_per_launch": round(ms, 5), "bound": "alu", "achieved": round(ach, 3),
                "peak": round(fp32_peak, 2), "unit": "TFLOP/s", "frac": round(ach / fp32_peak, 4),
                "edges_per_s": round(e / (ms * 1e-3), 1),
                "traffic": recorded_traffic(kernel, f"nequipl_{wl.name}")}

    line = {
        "metric": METRIC,
        "value": round(total_edges / (ms_step * 1e-3), 1),
        "unit": "edges/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded workload generator)",
        "config": {"workload": f"{wl.name}: {n} atoms, {e} edges, {wl.irreps}, SH lmax {wl.lmax}, "
                               f"r_cut {float(wl.r_cut)}, 8 Bessel",
                   "step": "neighbour list + CSR + fused forward + fused backward + forces",
                   "parallelism": f"replicas x{world}", "l2": "flushed (256 MB write) before every timed step"},
        "fwd_edges_per_s": round(total_edges / (ms_fwd * 1e-3), 1),
        "conv_fwd_bwd_edges_per_s": round(total_edges / ((ms_fwd + ms_bwd) * 1e-3), 1),
        "ms_fwd": round(ms_fwd, 5), "ms_bwd": round(ms_bwd, 5), "ms_graph": round(ms_graph, 5),
        "kernel_timing": f"median of {KERNEL_REPS} calls after {KERNEL_WARMUP} warm-up, L2 flushed before each",
        "roofline": roof(dominant, ms_bwd if dominant == "bwd" else ms_fwd),
        "roofline_fwd": roof("fwd", ms_fwd),
        "ms_weight_grad": round(ms_dw, 5),
        "roofline_weight_grad": roof("dw", ms_dw),
        "node_ladder": ladder_roof(ms_ladder),
        "node_ladder_full": ladder_full_roof(ms_ladder_full),
        "general_irreps_fwd": general_roof(ms_gen_fwd, "fwd"),
        "general_irreps_bwd": general_roof(ms_gen_bwd, "bwd"),
        "general_irreps_dw": general_roof(ms_gen_dw, "dw"),
        "workloads": others,
        "e2e": {"value": round(total_edges / (ms_e2e * 1e-3), 1), "unit": "edges/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step(info, n) * args.steps,
        "clocks": clocks,
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
    return line


# ---------------------------------------------------------------- other workloads

def measure_workload(name, dev, kernel_ms, fp32_peak, with_oracle=True):
    """Forward (and, except for the forward-only rank sweeps, backward) of one workload: graph build
    time, per-call device times, edges/s and FP32 roofline fractions of the whole calls."""
    import torch

    import equivariant_mlip_tensor_edge_b200 as etp
    import workloads

    wl = workloads.make(name)
    conv = etp.EdgeConv(wl.irreps, wl.lmax, wl.irreps, wl.n_basis, float(wl.r_cut))
    info = conv.info
    x = torch.from_numpy(wl.features()).to(dev)
    W = torch.from_numpy(wl.weights(conv.n_paths)).to(dev)
    if wl.given_receiver is not None:
        recv = torch.from_numpy(wl.given_receiver).to(dev)
        send = torch.from_numpy(wl.given_sender).to(dev)
        vec = torch.from_numpy(wl.given_edge_vec).to(dev)
        build = lambda: etp.build_csr(wl.n_nodes, recv, send, vec)
        graph_kind = "CSR from the given edge list"
    else:
        pos = torch.from_numpy(wl.pos).to(dev)
        build = lambda: etp.neighbors(pos, float(wl.r_cut), cell=wl.cell, pbc=wl.pbc)
        graph_kind = "neighbour list + CSR"
    gr = build()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    gr = build()
    torch.cuda.synchronize()
    ms_graph = 1000.0 * (time.perf_counter() - t0)
    ms_graph_dev = kernel_ms(build)
    e = gr.n_edges
    ws = torch.empty(max(conv.workspace_bytes(wl.n_nodes, e), 1), dtype=torch.uint8, device=dev)
    out = torch.empty((wl.n_nodes, info["dim_out"]), device=dev)
    ms_fwd = kernel_ms(lambda: conv.forward(gr, x, W, out=out, workspace=ws))
    cnt = algorithmic_counts(info, wl.n_nodes, e)
    ent = {"n_nodes": wl.n_nodes, "n_edges": e, "irreps": wl.irreps, "sh_lmax": wl.lmax,
           "ms_graph_wall": round(ms_graph, 3), "ms_graph": round(ms_graph_dev, 4), "graph": graph_kind,
           "ms_fwd": round(ms_fwd, 5), "fwd_edges_per_s": round(e / (ms_fwd * 1e-3), 1),
           "roofline_fwd_frac": round(cnt["fwd_flop"] / (ms_fwd * 1e-3) / 1e12 / fp32_peak, 4)}
    if not name.startswith("sweep"):
        g = torch.from_numpy(wl.cotangent()).to(dev)
        gx = torch.empty((wl.n_nodes, info["dim_in"]), device=dev)
        gv = torch.empty((e, 3), device=dev)
        ms_bwd = kernel_ms(lambda: conv.backward(gr, x, W, g, grad_x=gx, grad_vec=gv, workspace=ws))
        ent.update({"ms_bwd": round(ms_bwd, 5),
                    "fwd_bwd_edges_per_s": round(e / ((ms_fwd + ms_bwd) * 1e-3), 1),
                    "roofline_bwd_frac": round(cnt["bwd_flop"] / (ms_bwd * 1e-3) / 1e12 / fp32_peak, 4)})
    ent["roofline_peak"] = {"unit": "TFLOP/s", "value": round(fp32_peak, 2), "bound": "alu"}
    if with_oracle:
        ent["cpu_baseline"] = oracle_workload_sample(wl, ORACLE_SAMPLE[name], backward=not name.startswith("sweep"))
    return ent


def oracle_workload_sample(wl, n_recv, backward=True):
    """The float64 oracle, as it stands, on n_recv sampled receivers of the workload (one BLAS
    thread): their neighbour rows (or given edges), the forward, and the VJP."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    from oracle.conv import ConvSpec, conv_forward, conv_vjp
    from oracle.graph import neighbors

    spec = ConvSpec(wl.irreps, wl.lmax, wl.irreps, wl.n_basis, float(wl.r_cut))
    x, W = wl.features(), wl.weights(len(spec.paths))
    n_recv = min(n_recv, wl.n_nodes)
    sample = sorted(np.random.default_rng(0).choice(wl.n_nodes, size=n_recv, replace=False).tolist())
    with threadpool_limits(1):
        t0 = time.perf_counter()
        if wl.given_receiver is not None:
            order = np.lexsort((wl.given_sender, wl.given_receiver))
            r, s_, v = wl.given_receiver[order], wl.given_sender[order], wl.given_edge_vec[order]
            keep = np.isin(r, sample)
            r, s_, v = r[keep], s_[keep], v[keep]
        else:
            rows = neighbors(wl.pos, wl.cell, wl.pbc, wl.r_cut, receivers=sample)
            r, s_, v = rows["receiver"], rows["sender"], rows["edge_vec"]
        rp = np.zeros(wl.n_nodes + 1, dtype=np.int64)
        np.add.at(rp, np.asarray(r) + 1, 1)
        rp = np.cumsum(rp)
        conv_forward(spec, rp, s_, v, x, W, receivers=sample)
        if backward:
            conv_vjp(spec, rp, s_, v, x, W, wl.cotangent())
        dt = time.perf_counter() - t0
    edges = len(s_)
    return {"value": round(edges / dt, 1), "unit": "edges/s", "cores": 1, "host_cores": os.cpu_count(),
            "kind": "oracle",
            "sample": f"{n_recv} of {wl.n_nodes} receivers ({edges} edges): "
                      f"{'neighbour rows' if wl.given_receiver is None else 'given edges'}, forward"
                      f"{', VJP' if backward else ''} in float64 numpy on one BLAS thread, {dt:.2f} s",
            "seconds": round(dt, 3)}


# ---------------------------------------------------------------- oracle (CPU) timing

def _oracle_sample_step(wl, sample):
    import numpy as np

    from oracle.conv import ConvSpec, conv_forward, conv_vjp
    from oracle.graph import forces_from_edge_grads, neighbors

    spec = ConvSpec(wl.irreps, wl.lmax, wl.irreps, wl.n_basis, float(wl.r_cut))
    x, W, g = wl.features(), wl.weights(len(spec.paths)), wl.cotangent()
    rows = neighbors(wl.pos, wl.cell, wl.pbc, wl.r_cut, receivers=sample)
    row_ptr = np.zeros(wl.n_nodes + 1, dtype=np.int64)
    np.add.at(row_ptr, rows["receiver"] + 1, 1)
    row_ptr = np.cumsum(row_ptr)
    conv_forward(spec, row_ptr, rows["sender"], rows["edge_vec"], x, W, receivers=sample)
    _, gv = conv_vjp(spec, row_ptr, rows["sender"], rows["edge_vec"], x, W, g)
    forces_from_edge_grads(gv, rows["receiver"], rows["sender"], wl.n_nodes)
    return len(rows["sender"])


def cpu_baseline(wl, budget_s=15.0, steps=1):
    """The float64 oracle, as it stands, on a bounded sample of receivers; one BLAS thread."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    frac = 0.25
    n_s = max(1, int(wl.n_nodes * frac))
    sample = sorted(np.random.default_rng(0).choice(wl.n_nodes, size=n_s, replace=False).tolist())
    with threadpool_limits(1):
        t0 = time.perf_counter()
        edges = 0
        for _ in range(steps):
            edges += _oracle_sample_step(wl, sample)
        dt = time.perf_counter() - t0
    return {"value": round(edges / dt, 1), "unit": "edges/s", "cores": 1, "host_cores": os.cpu_count(),
            "kind": "oracle",
            "sample": f"{n_s} of {wl.n_nodes} receivers ({edges // steps} edges): neighbour rows, forward, VJP, "
                      f"forces in float64 numpy, {steps} step(s), {dt:.1f} s",
            "seconds": round(dt, 3)}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import workloads
    wl = workloads.make(args.workload)
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up state; kept for the CLI contract
    cb = cpu_baseline(wl, budget_s=args.cpu_budget, steps=max(1, args.steps))
    ms = 1000.0 * cb["seconds"] / max(1, args.steps)
    return {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "edges/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded workload generator)",
            "config": {"workload": wl.name, "step": "neighbour rows + forward + VJP + forces (float64 oracle)",
                       "parallelism": "host cores, rank 0 only"},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="etp", choices=["etp", "reference"])
    ap.add_argument("--workload", default="diamond1k")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true", help="skip the per-workload entries")
    ap.add_argument("--kernel-reps", type=int, default=KERNEL_REPS,
                    help="timed calls per kernel timing (fewer only for profiler runs)")
    ap.add_argument("--kernel-warmup", type=int, default=KERNEL_WARMUP)
    args = ap.parse_args()
    set_kernel_timing(args.kernel_reps, args.kernel_warmup)
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
