"""Benchmark of the SSD forward scan on B200: one JSON line on stdout (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one ssd_forward call -- the whole hot path (ssd_chunk_cumsum,
ssd_chunk_state, ssd_state_passing, ssd_chunk_scan; on this layer the last
three run as the library's single-pass kernel) -- over one batch of the
Mamba-2-2.7B-shaped layer (B=4, T=4096, H=80, P=64, N=128, G=1, chunk 256,
bf16 x/B/C, fp32 dt/A/D, final state returned), seeded synthetic inputs resident
in HBM.  Every step's inputs and outputs exceed L2 (x and y are 168 MB each,
L2 is 126 MB), so steps run back to back without a flush.

Multi-GPU (torchrun, one process per GPU): the path is not sharded; every rank
runs an independent replica of the same workload ("weak" scaling) and the
time is the max over ranks.  --impl reference times the fp64 CPU oracle on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from structured_state_space_mamba_b200.inputs import WORKLOADS, make_workload  # noqa: E402

METRIC = "SSD scan tokens/sec on 1 B200 and % of bf16 tensor-core roofline"
UNIT = "tokens/s"
SPEC_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
THROTTLE_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
                 0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
                 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
                 0x100: "display_clock_setting"}


# ---------------------------------------------------------------------------
# algorithmic work (chunked algorithm; compulsory bytes only)
# ---------------------------------------------------------------------------
# DRAM bytes (read + write) of one launch of the dominant kernel on a workload,
# from one ncu capture of the current kernel (dram__bytes_read.sum +
# dram__bytes_write.sum); workloads without such a capture report None.
# Keyed by (workload, kernel, library version): a capture stands only for the
# build it was taken from, so a rebuilt kernel reports traffic None until it is
# captured again.
NCU_TRAFFIC = {
    # profiles/full_chunk_fused_mamba2_2p7b.md: 187.87 MB read + 139.70 MB written
    ("mamba2_2p7b", "ssd_chunk_fused", "ssd-b200 0.3.1 sm_100a"): 327_571_456,
    # profiles/sol_kernels_long_g8.md (presolved single pass): 564.46 MB read + 236.48 MB written
    ("long_g8", "ssd_chunk_fused", "ssd-b200 0.3.1 sm_100a"): 800_936_704,
}


def ncu_traffic(workload, kernel):
    from structured_state_space_mamba_b200 import binding
    return NCU_TRAFFIC.get((workload, kernel, binding.version()))


def max_over_ranks(value, world, device):
    """The largest of every rank's `value` (a time); every rank gets it.  One
    all-reduce over the job's process group (NCCL on GPUs, gloo on CPUs)."""
    if world == 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(world, units_per_rank_step, steps, ms):
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (weak scaling: every rank does the same work)."""
    return world * units_per_rank_step * steps / (ms * 1e-3)


def work_model(cfg, final_state=True, lay=None):
    B, T, H, P, N, G, Q = (cfg[k] for k in ("batch", "seqlen", "nheads", "headdim", "dstate",
                                            "ngroups", "chunk_len"))
    nc = T // Q
    esz = 2 if cfg["dtype"] == "bf16" else 4
    flops_bch = Q * (Q + 1) * P + 4 * Q * N * P          # masked product + state + C.s_in
    flops_bcg = Q * (Q + 1) * N                          # causal C B^T, shared by H/G heads
    flops = B * nc * (H * flops_bch + G * flops_bcg)
    x_bytes = B * T * H * P * esz
    bc_bytes = 2 * B * T * G * N * esz
    dt_bytes = B * T * H * 4
    state_bytes = B * H * P * N * 4
    comp = (2 * x_bytes + bc_bytes + dt_bytes + 2 * H * 4
            + (state_bytes if cfg.get("init_state") else 0)
            + (state_bytes if final_state else 0))
    if cfg.get("block"):
        # the block's neighbours: z in, the norm weight [H*P] and dt_bias [H]
        comp += x_bytes + H * P * 4 + H * 4
    # per-kernel algorithmic bytes (what each kernel must read and write, with the
    # element sizes of this call's workspace layout)
    st_elems = B * nc * H * P * N
    lq = B * H * nc * Q * 4                               # one fp32 [B,H,nc,Q] array
    s_sz = 2 if (lay is None or lay.states_dtype == 1) else 4
    sin_sz = 2 if (lay is None or lay.s_in_dtype == 1) else 4
    fused = bool(lay is not None and lay.fused_state)
    # the chunk-wide scan (one launch more than the four-stage sequence) reads l
    # and the per-token factors g [B,H,nc,Q+4] instead of l, dtq and beta
    chunkwide = bool(lay is not None and lay.launches == (3 if fused else 4) + 1)
    gq_bytes = B * H * nc * (Q + 4) * 4
    h0_bytes = state_bytes if cfg.get("init_state") else 0
    fin_bytes = state_bytes if final_state else 0
    tail = 1 if lay is not None and T % lay.chunk_len else 0  # the ragged tail's own launch
    if lay is not None and getattr(lay, "single_pass", 0) and lay.launches - tail == 5:
        # presolved single pass: cumsum (fused mode, plus w and alpha); the range
        # states: x, B, w, alpha, h0 -> one partial state per CTA, chained along
        # each chain (small); the single pass from those states, then the
        # block-factored scan of the listed tiles
        pre_bytes = min(B * (H // 2) * nc, 148) * 128 * N * 4  # one state per CTA of the single pass
        per_kernel = {
            "ssd_chunk_cumsum": dt_bytes + H * 4 + 2 * lq + gq_bytes + B * H * nc * 4,
            "ssd_range_states": x_bytes + bc_bytes // 2 + lq + B * H * nc * 4 + h0_bytes + 3 * pre_bytes,
            "ssd_chunk_fused": (2 * x_bytes + bc_bytes + lq + gq_bytes + H * 4 + h0_bytes + fin_bytes
                                + pre_bytes),
        }
        per_kernel_comp = {
            "ssd_chunk_cumsum": dt_bytes + H * 4,
            "ssd_range_states": 0,
            "ssd_chunk_fused": 2 * x_bytes + bc_bytes + H * 4 + h0_bytes + fin_bytes,
        }
        per_kernel_flops = {"ssd_range_states": 2 * B * nc * H * Q * N * P, "ssd_chunk_fused": flops}
        return dict(flops=flops, bytes=comp, per_kernel_bytes=per_kernel,
                    per_kernel_comp=per_kernel_comp, per_kernel_flops=per_kernel_flops,
                    stages=("ssd_chunk_cumsum", "ssd_range_states", None, "ssd_chunk_fused"))
    if lay is not None and getattr(lay, "single_pass", 0):
        # cumsum (fused mode): dt, A -> l and g (dtq and beta only for chunks with
        # a steep tile); the single-pass kernel: x, B, C, l, g, D, h0 -> y, final
        # (its per-(b, h) state slots stay in L2: B*H*P*N*4 bytes, each written
        # and read once per chunk); the block-factored scan: only listed tiles
        per_kernel = {
            "ssd_chunk_cumsum": dt_bytes + H * 4 + lq + gq_bytes,
            "ssd_chunk_fused": (2 * x_bytes + bc_bytes + lq + gq_bytes + H * 4 + h0_bytes + fin_bytes),
            "ssd_chunk_scan_steep": 0,
        }
        per_kernel_comp = {
            "ssd_chunk_cumsum": dt_bytes + H * 4,
            "ssd_chunk_fused": 2 * x_bytes + bc_bytes + H * 4 + h0_bytes + fin_bytes,
            "ssd_chunk_scan_steep": 0,
        }
        per_kernel_flops = {"ssd_chunk_fused": flops}
        return dict(flops=flops, bytes=comp, per_kernel_bytes=per_kernel,
                    per_kernel_comp=per_kernel_comp, per_kernel_flops=per_kernel_flops,
                    stages=("ssd_chunk_cumsum", "ssd_chunk_fused", None, "ssd_chunk_scan_steep"))
    per_kernel = {
        # dt, A -> l, w, dtq, beta, alpha (and g for the chunk-wide scan)
        "ssd_chunk_cumsum": dt_bytes + H * 4 + 4 * lq + B * H * nc * 4 + (gq_bytes if chunkwide else 0),
        # x, B, w -> S  (fused: x, B, w, alpha, h0 -> s_in, final)
        "ssd_chunk_state": (x_bytes + bc_bytes // 2 + lq + B * H * nc * 4 + h0_bytes
                            + st_elems * sin_sz + fin_bytes) if fused
                           else (x_bytes + bc_bytes // 2 + lq + st_elems * s_sz),
        "ssd_state_passing": 0 if fused else (st_elems * s_sz + B * H * nc * 4 + h0_bytes
                                              + st_elems * sin_sz + fin_bytes),
        # x, B, C, l, (g | dtq, beta), s_in, D -> y
        "ssd_chunk_scan": (2 * x_bytes + bc_bytes + (lq + gq_bytes if chunkwide else 3 * lq)
                           + st_elems * sin_sz + H * 4),
    }
    # the compulsory bytes (above) that each kernel moves itself: the roofline
    # fraction of a kernel counts only these; workspace traffic is its loss
    per_kernel_comp = {
        "ssd_chunk_cumsum": dt_bytes + H * 4,
        "ssd_chunk_state": x_bytes + bc_bytes // 2 + ((h0_bytes + fin_bytes) if fused else 0),
        "ssd_state_passing": 0 if fused else h0_bytes + fin_bytes,
        "ssd_chunk_scan": 2 * x_bytes + bc_bytes + H * 4,
    }
    per_kernel_flops = {
        "ssd_chunk_state": 2 * B * nc * H * Q * N * P,
        "ssd_chunk_scan": B * nc * (H * (Q * (Q + 1) * P + 2 * Q * N * P) + G * flops_bcg),
    }
    return dict(flops=flops, bytes=comp, per_kernel_bytes=per_kernel,
                per_kernel_comp=per_kernel_comp, per_kernel_flops=per_kernel_flops,
                stages=("ssd_chunk_cumsum", "ssd_chunk_state", "ssd_state_passing", "ssd_chunk_scan"))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(SPEC_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
def gpu_identity(device_index):
    """nvidia-smi's id of the torch device: its UUID ("GPU-..."), which names the
    same physical GPU whatever CUDA_VISIBLE_DEVICES maps (nvidia-smi's own
    indices follow PCI order and ignore it); the PCI bus id if no UUID is known."""
    import torch
    p = torch.cuda.get_device_properties(device_index)
    u = str(getattr(p, "uuid", "") or "")
    if u:
        return u if u.startswith("GPU-") else "GPU-" + u
    return "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)


class ClockSampler:
    """Samples the SM clock and the clock-event reasons of ONE GPU, named by its
    nvidia-smi id (gpu_identity), while the timed region runs."""

    def __init__(self, gpu_id):
        self.proc = None
        self.gpu_id = str(gpu_id)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id,
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        return False

    def summary(self):
        if self.proc is None or not getattr(self, "out", None):
            return None
        sm, mx, reasons = [], [], set()
        for line in self.out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 4:
                continue
            try:
                s, m = float(parts[0]), float(parts[1])
                bits = int(parts[3], 16) if parts[3].startswith("0x") else int(parts[3])
            except ValueError:
                continue
            if bits & 0x1:  # idle samples say nothing about the load
                continue
            sm.append(s)
            mx.append(m)
            for bit, name in THROTTLE_BITS.items():
                if bits & bit:
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm), "gpu": self.gpu_id}


# ---------------------------------------------------------------------------
# oracle leg (CPU)
# ---------------------------------------------------------------------------
def oracle_sample(inp, tokens, batches=1):
    """Run the oracle over the first `tokens` tokens of `batches` batch rows
    (all heads); returns (seconds, tokens processed, threads)."""
    import oracle
    sl = slice(0, tokens)
    bs = slice(0, batches)
    args = [inp.x[bs, sl], inp.dt[bs, sl], inp.A, inp.B[bs, sl], inp.C[bs, sl]]
    h0 = None if inp.h0 is None else inp.h0[bs]
    t0 = time.perf_counter()
    oracle.ssd_recurrent(*args, D=inp.D, h0=h0)
    return time.perf_counter() - t0, tokens * batches, oracle.default_threads()


def cpu_baseline(inp, budget_s=12.0):
    import oracle  # noqa: F401  (builds the C oracle if needed)
    T = inp.x.shape[1]
    tokens = min(T, 512)
    sec, tok, th = oracle_sample(inp, tokens)
    # grow the sample to roughly budget_s of CPU work
    scale = max(1, int(budget_s / max(sec, 1e-3)))
    bmax = inp.x.shape[0]
    tokens2 = min(T, tokens * scale)
    batches = min(bmax, max(1, (tokens * scale) // T)) if tokens2 == T else 1
    sec, tok, th = oracle_sample(inp, tokens2, batches)
    return {"value": tok / sec, "unit": UNIT, "cores": th, "kind": "oracle",
            "sample": f"fp64 recurrence over the first {tokens2} tokens x {batches} batch row(s), "
                      f"all {inp.x.shape[2]} heads ({tok} tokens, {sec:.1f} s on {th} threads)"}


def run_reference(args, cfg, rank):
    if rank != 0:
        return
    inp = make_workload(args.workload)
    T = inp.x.shape[1]
    tokens = min(T, args.ref_tokens)
    for _ in range(args.warmup):
        oracle_sample(inp, tokens)
    secs = []
    th = 1
    for _ in range(args.steps):
        s, _, th = oracle_sample(inp, tokens)
        secs.append(s)
    total = sum(secs)
    value = tokens * args.steps / total
    sample = (f"each step: fp64 recurrence over the first {tokens} of {T} tokens of batch row 0, "
              f"all {inp.x.shape[2]} heads")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": config_block(cfg, args.workload,
                                   l2_policy(cfg, device_l2_bytes(int(os.environ.get("LOCAL_RANK", "0"))))[1]),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": th, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


L2_FALLBACK_BYTES = 126 * 1000 * 1000


def l2_policy(cfg, l2_bytes):
    """(flush, note): a workload whose x (and y) each exceed L2 is timed back to
    back; a smaller one gets L2 flushed before every timed step, outside the
    events that time the step."""
    esz = 2 if cfg["dtype"] == "bf16" else 4
    x_bytes = cfg["batch"] * cfg["seqlen"] * cfg["nheads"] * cfg["headdim"] * esz
    if x_bytes > l2_bytes:
        return False, (f"no flush: inputs larger than L2 (x and y {x_bytes / 1e6:.0f} MB each, "
                       f"L2 {l2_bytes / 1e6:.0f} MB)")
    return True, (f"L2 flushed before every timed step by a {2 * l2_bytes / 1e6:.0f} MB write outside "
                  f"the step's events (x and y {x_bytes / 1e6:.0f} MB each, L2 {l2_bytes / 1e6:.0f} MB)")


def device_l2_bytes(device_index=0):
    """L2 size of the GPU the run uses (the fallback when no GPU is visible);
    both arms build config.l2 from it, so identical workloads get identical
    config blocks."""
    try:
        import torch
        if torch.cuda.is_available():
            return int(getattr(torch.cuda.get_device_properties(device_index), "L2_cache_size", 0)
                       or L2_FALLBACK_BYTES)
    except Exception:  # noqa: BLE001 -- the note is informational
        pass
    return L2_FALLBACK_BYTES


def config_block(cfg, name, l2_note=None):
    return {"workload": (f"{name}: B={cfg['batch']} T={cfg['seqlen']} H={cfg['nheads']} "
                         f"P={cfg['headdim']} N={cfg['dstate']} G={cfg['ngroups']} "
                         f"chunk={cfg['chunk_len']} {cfg['dtype']}"),
            "batch": cfg["batch"], "seqlen": cfg["seqlen"], "nheads": cfg["nheads"],
            "headdim": cfg["headdim"], "dstate": cfg["dstate"], "ngroups": cfg["ngroups"],
            "chunk_len": cfg["chunk_len"], "init_state": bool(cfg.get("init_state")),
            "final_state": bool(cfg.get("final_state", True)),
            "l2": l2_note if l2_note is not None else l2_policy(cfg, L2_FALLBACK_BYTES)[1],
            "parallelism": "replicas",
            **({"block": "softplus(dt + dt_bias), y * silu(z), RMSNorm over H*P"}
               if cfg.get("block") else {})}


# ---------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------
def run_gpu(args, cfg, rank, world, local_rank):
    import torch

    from structured_state_space_mamba_b200 import binding

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    inp = make_workload(args.workload, **({"batch": cfg["batch"]} if args.batch else {}))
    tt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    host = dict(x=(inp.x, tt), dt=(inp.dt, torch.float32), A=(inp.A, torch.float32),
                B=(inp.B, tt), C=(inp.C, tt), D=(inp.D, torch.float32))
    if inp.h0 is not None:
        host["init_state"] = (inp.h0, torch.float32)
    # pinned host copies (storage dtype) for the end-to-end leg
    pinned = {k: torch.from_numpy(v).to(t).pin_memory() for k, (v, t) in host.items()}
    d = {k: v.to(dev, non_blocking=False) for k, v in pinned.items()}
    want_final = bool(cfg.get("final_state", True))
    y = torch.empty_like(d["x"])
    fin = (torch.empty((inp.x.shape[0], inp.x.shape[2], inp.x.shape[3], inp.B.shape[3]),
                       dtype=torch.float32, device=dev) if want_final else None)
    dims = binding.make_dims(*inp.x.shape[:2], inp.x.shape[2], inp.x.shape[3], inp.B.shape[3],
                             inp.B.shape[2], inp.dtype)
    lay = binding.workspace_layout(dims, inp.chunk_len)
    ws = torch.empty(lay.total_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    block = bool(cfg.get("block"))
    if block:
        # the block's raw inputs: dt_raw = softplus^-1(dt) - dt_bias, so the scan
        # sees the workload's own step sizes; z ~ N(0, 1); weight 1 + 0.1 N(0, 1)
        rng = np.random.default_rng(3000)
        bias = rng.uniform(-0.5, 0.5, size=inp.A.shape).astype(np.float32)
        dt_raw = (np.log(np.expm1(inp.dt.astype(np.float64))) - bias[None, None, :]).astype(np.float32)
        zh = rng.standard_normal(inp.x.shape).astype(np.float32)
        wn = (1.0 + 0.1 * rng.standard_normal(inp.x.shape[2] * inp.x.shape[3])).astype(np.float32)
        pinned["dt"] = torch.from_numpy(dt_raw).pin_memory()
        pinned["z"] = torch.from_numpy(zh).to(tt).pin_memory()
        d["dt"] = pinned["dt"].to(dev)
        d["z"] = pinned["z"].to(dev)
        d["dt_plain"] = torch.from_numpy(inp.dt).to(dev)
        bias_d = torch.from_numpy(bias).to(dev)
        wn_d = torch.from_numpy(wn).to(dev)
        ws_block = torch.empty(binding.block_workspace_bytes(dims, inp.chunk_len, True),
                               dtype=torch.uint8, device=dev)

    def step(stage=None):
        if block and stage is None:
            binding.forward_block(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"],
                                  chunk_len=inp.chunk_len, init_state=d.get("init_state"),
                                  dt_bias=bias_d, dt_softplus=True, z=d["z"], norm_weight=wn_d,
                                  out=y, final_out=fin, workspace=ws_block)
            return
        binding.forward(d["x"], d["dt_plain"] if block else d["dt"], d["A"], d["B"], d["C"], D=d["D"],
                        chunk_len=inp.chunk_len, init_state=d.get("init_state"), out=y,
                        final_out=fin, workspace=ws, stage=stage)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    def max_ms(v):
        return max_over_ranks(v, world, dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- the step as a CUDA graph (one ssd_forward_ws call, captured) -------
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            with torch.cuda.graph(graph, stream=cap):
                step()
        stream.wait_stream(cap)
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()

    l2_bytes = device_l2_bytes(local_rank)
    flush, l2_note = l2_policy(cfg, l2_bytes)
    flush_buf = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev) if flush else None

    def timed(run_step):
        if flush:
            # each step timed on its own, after a write that evicts L2
            pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(args.steps)]
            barrier()
            torch.cuda.synchronize()
            for a, b in pairs:
                flush_buf.zero_()
                a.record(stream)
                run_step()
                b.record(stream)
            torch.cuda.synchronize()
            barrier()
            return max_ms(sum(a.elapsed_time(b) for a, b in pairs))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            run_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return max_ms(e0.elapsed_time(e1))

    # ---- timed region: K back-to-back steps -------------------------------
    with ClockSampler(gpu_identity(local_rank)) as clk:
        ms_direct = timed(step)
        ms_graph = timed(graph.replay) if graph is not None else None
    clocks = clk.summary()
    if ms_graph is not None and ms_graph < ms_direct:
        ms_total, launch_mode = ms_graph, "cuda-graph replay of one ssd_forward_ws call per step"
    else:
        ms_total, launch_mode = ms_direct, "one ssd_forward_ws call per step"
    del graph

    # ---- per-kernel durations: the same steps, one stage per launch ---------
    # A GPU-side sleep before each step lets the host enqueue all four stages
    # (and the events between them) first, so no host launch gap lands inside
    # an event pair.  Stage names follow the call's layout (the single-pass
    # layout runs stages 1-3 of the four-kernel sequence as one kernel, plus the
    # block-factored scan of the listed steep tiles).
    names = work_model(cfg, final_state=want_final, lay=lay)["stages"]
    nst = len(names)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for k in range(args.steps):
        torch.cuda._sleep(3_000_000)
        ev[k][0].record(stream)
        for s in range(nst):
            step(stage=s)
            ev[k][s + 1].record(stream)
    torch.cuda.synchronize()
    kern_ms = {names[s]: statistics.mean(ev[k][s].elapsed_time(ev[k][s + 1]) for k in range(args.steps))
               for s in range(nst) if names[s] is not None}
    if block:
        # the block's gate and norm (one kernel after the scan): the block step
        # minus the plain scan's stages, on the same inputs
        ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        torch.cuda.synchronize()
        for a, b in ev2:
            torch.cuda._sleep(1_000_000)
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        blk = statistics.mean(a.elapsed_time(b) for a, b in ev2)
        kern_ms["ssd_gate_norm"] = max(blk - sum(kern_ms.values()), 1e-6)
    barrier()

    # ---- end to end through the public call, host buffers ------------------
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    fin_host = torch.empty(fin.shape, dtype=fin.dtype).pin_memory() if fin is not None else None
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = y_host.numel() * y_host.element_size() + (
        fin_host.numel() * fin_host.element_size() if fin_host is not None else 0)

    def e2e_step():
        for k, v in pinned.items():
            d[k].copy_(v, non_blocking=True)
        step()
        y_host.copy_(y, non_blocking=True)
        if fin_host is not None:
            fin_host.copy_(fin, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_ms(f0.elapsed_time(f1))
    barrier()

    if rank != 0:
        return
    tokens_step = inp.x.shape[0] * inp.x.shape[1]
    value = job_rate(world, tokens_step, args.steps, ms_total)
    wm = work_model(cfg, final_state=want_final, lay=lay)
    if block:
        gn = 3 * inp.x.size * (2 if inp.dtype == "bf16" else 4) + inp.x.shape[2] * inp.x.shape[3] * 4
        wm["per_kernel_comp"]["ssd_gate_norm"] = gn
        wm["per_kernel_bytes"]["ssd_gate_norm"] = gn
    peaks, peak_src = load_peaks()
    top = max(kern_ms, key=kern_ms.get)
    bound = "hbm"
    t_step = ms_total / args.steps * 1e-3
    # the kernel's time inside the timed step: its share of the per-stage event
    # times applied to the step (stage-by-stage launches carry launch gaps that
    # the graph-replayed step does not, so their sum exceeds the step)
    share = kern_ms[top] / sum(kern_ms.values())
    t_top = share * t_step
    achieved = wm["per_kernel_comp"][top] / t_top / 1e9
    peak = peaks["hbm_gbs"]
    t_roof = max(wm["flops"] / (peaks["bf16_tflops"] * 1e12), wm["bytes"] / (peaks["hbm_gbs"] * 1e9))
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": inp.dtype, "data": "synthetic",
        "config": config_block(cfg, args.workload, l2_note),
        "roofline": {"bound": bound, "kernel": top, "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None if args.batch is not None else ncu_traffic(args.workload, top),
                     "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)",
                     "bytes": "compulsory bytes the kernel moves (inputs it reads, outputs it "
                              "writes); workspace traffic counts against it",
                     "compulsory_bytes": wm["per_kernel_comp"][top],
                     "kernel_us_in_step": t_top * 1e6, "kernel_share_of_step": share,
                     "bytes_incl_workspace": wm["per_kernel_bytes"][top],
                     "frac_incl_workspace": wm["per_kernel_bytes"][top] / t_top / 1e9 / peak},
        "path_roofline": {"t_roof_us": t_roof * 1e6, "t_step_us": t_step * 1e6,
                          "frac": t_roof / t_step, "flops": wm["flops"],
                          "compulsory_bytes": wm["bytes"],
                          "peaks": f"{peak_src}: hbm {peaks['hbm_gbs']} GB/s, "
                                   f"bf16 {peaks['bf16_tflops']} TF/s"},
        "kernels_us": {k: v * 1e3 for k, v in kern_ms.items()},
        "launch": launch_mode + (" (ssd_forward_block)" if block else ""),
        "ms_per_step_direct_calls": ms_direct / args.steps,
        "gpu_launches": args.steps * (lay.launches + (1 if block else 0)),
        "tensor_core": bool(lay.tensor_core),
        "fused_state": bool(lay.fused_state),
        "single_pass": bool(lay.single_pass),
        "scan_engine": binding.SCAN_ENGINES.get(lay.scan_engine, lay.scan_engine),
        "e2e": {"value": job_rate(world, tokens_step, args.steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inp)
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# backward (ssd_backward): the gradients of every input for one batch
# ---------------------------------------------------------------------------
BACKWARD_METRIC = "SSD backward tokens/sec on 1 B200 (gradients of every input) and % of HBM roofline"


def backward_launches(inp):
    """Kernels one ssd_backward call launches, following the choices it makes:
    the input preparation (2 kernels, plus fp32 copies of x, B and C for bf16
    inputs and of dy when the transposed scans run in fp32), the transposed
    dfinal and h0, the scans of K and h (fp32, 64-token chunks unless that plan
    is refused, then the caller's length), the transposed scans (per 64-wide
    dstate slice on the bf16 tensor-core plans where they apply, else one fp32
    scan each) and the five kernels that finish the gradients."""
    from structured_state_space_mamba_b200 import binding
    B_, T, H, P = inp.x.shape
    G, N = inp.B.shape[2], inp.B.shape[3]
    bf16 = inp.dtype == "bf16"
    f32 = binding.make_dims(B_, T, H, P, N, G, "f32")
    try:
        scan = binding.workspace_layout(f32, 64).launches
    except binding.SSDError:
        scan = binding.workspace_layout(f32, inp.chunk_len).launches
    scan_bf16 = False
    if bf16 and P == 64 and N % 64 == 0:
        lay = binding.workspace_layout(binding.make_dims(B_, T, H, 64, P, H, "bf16"), inp.chunk_len)
        scan_bf16 = binding.SCAN_ENGINES.get(lay.scan_engine) != "simt"
    if scan_bf16:
        transposed = 2 * (N // 64) * lay.launches
    else:
        transposed = 2 * binding.workspace_layout(binding.make_dims(B_, T, H, N, P, H, "f32"), inp.chunk_len).launches
    prep = 2 + (3 if bf16 else 0) + (1 if bf16 and not scan_bf16 else 0)
    states = 1 + (1 if inp.h0 is not None else 0)  # dfinal (always given here) and h0
    return prep + states + 2 * scan + transposed + 5


def run_backward(args, cfg, rank, world, local_rank):
    import torch
    from structured_state_space_mamba_b200 import binding
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    inp = make_workload(args.workload, **({"batch": cfg["batch"]} if args.batch else {}))
    tt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    rng = np.random.default_rng(4000 + rank)
    dy_h = rng.standard_normal(inp.x.shape).astype(np.float32)
    fin_h = rng.standard_normal((inp.x.shape[0], inp.x.shape[2], inp.x.shape[3], inp.B.shape[3])).astype(np.float32)
    host = dict(x=(inp.x, tt), dt=(inp.dt, torch.float32), A=(inp.A, torch.float32), B=(inp.B, tt),
                C=(inp.C, tt), D=(inp.D, torch.float32), dy=(dy_h, tt), dfin=(fin_h, torch.float32))
    if inp.h0 is not None:
        host["h0"] = (inp.h0, torch.float32)
    pinned = {k: torch.from_numpy(np.ascontiguousarray(v)).to(ty).pin_memory() for k, (v, ty) in host.items()}
    d = {k: v.to(dev) for k, v in pinned.items()}
    stream = torch.cuda.current_stream(dev)
    outs = {}

    def step():
        outs["g"] = binding.backward(d["x"], d["dt"], d["A"], d["B"], d["C"], d["dy"], D=d["D"],
                                     chunk_len=inp.chunk_len, init_state=d.get("h0"), dfinal_state=d["dfin"])

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_identity(local_rank)) as clk:
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    clocks = clk.summary()
    # end to end: inputs and dy in from pinned host memory, every gradient back
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    d2h = 0
    for _ in range(args.steps):
        for k, v in pinned.items():
            d[k].copy_(v, non_blocking=True)
        step()
        d2h = 0
        for g in outs["g"].values():
            if g is not None:
                g.cpu()
                d2h += g.numel() * g.element_size()
    f1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, dev)
    if rank != 0:
        return
    B_, T, H, P = inp.x.shape
    G, N = inp.B.shape[2], inp.B.shape[3]
    esz = 2 if inp.dtype == "bf16" else 4
    st = B_ * H * P * N * 4
    # compulsory bytes: x, dy, B, C, dt, A, D, h0, dfinal in; dx, dB, dC, ddt, dA, dD, dinit out
    comp = (3 * B_ * T * H * P * esz + 4 * B_ * T * G * N * esz + 2 * B_ * T * H * 4 + 4 * H * 4
            + (2 * st if inp.h0 is not None else 0) + st)
    t_step = ms / args.steps * 1e-3
    peaks, peak_src = load_peaks()
    achieved = comp / t_step / 1e9
    line = {
        "metric": BACKWARD_METRIC, "value": job_rate(world, B_ * T, args.steps, ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": inp.dtype,
        "data": "synthetic", "config": dict(config_block(cfg, args.workload), backward=True),
        "roofline": {"bound": "hbm", "kernel": "ssd_backward (whole call)", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": None, "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)",
                     "compulsory_bytes": comp},
        "launch": "one ssd_backward call per step (four fp32 scans and the element-wise kernels)",
        "gpu_launches": args.steps * backward_launches(inp),
        "e2e": {"value": job_rate(world, B_ * T, args.steps, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# decode step (ssd_step): one token per (batch, head) on a resident state
# ---------------------------------------------------------------------------
DECODE = dict(batch=64, nheads=80, headdim=64, dstate=128, ngroups=1, dtype="bf16")
DECODE_METRIC = "SSD decode-step tokens/sec on 1 B200 and % of HBM roofline"


def decode_inputs(cfg, seed=2000):
    """One decode token per batch row, drawn like the scan's inputs, and a state
    drawn N(0, 0.1^2) (resident on the device between steps)."""
    from structured_state_space_mamba_b200.inputs import make_inputs
    inp = make_inputs(cfg["batch"], 1, cfg["nheads"], cfg["headdim"], cfg["dstate"], cfg["ngroups"], 1,
                      dtype=cfg["dtype"], seed=seed, init_state=True, h0_std=0.1)
    return dict(x=inp.x[:, 0], dt=inp.dt[:, 0], A=inp.A, B=inp.B[:, 0], C=inp.C[:, 0], D=inp.D,
                state=inp.h0)


def decode_cpu_baseline(v, budget_s=8.0):
    """The oracle's fp64 step on the host, repeated for about budget_s."""
    import oracle
    n, t0 = 0, time.perf_counter()
    state = v["state"]
    while time.perf_counter() - t0 < budget_s:
        _, state = oracle.ssd_step(state, v["x"], v["dt"], v["A"], v["B"], v["C"], D=v["D"])
        n += 1
    sec = time.perf_counter() - t0
    bsz = v["x"].shape[0]
    return {"value": n * bsz / sec, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"fp64 numpy step over the full decode shape, {n} steps in {sec:.1f} s"}


def run_decode(args, rank, world, local_rank):
    import torch
    from structured_state_space_mamba_b200 import binding
    cfg = dict(DECODE)
    if args.batch is not None:
        cfg["batch"] = args.batch
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    v = decode_inputs(cfg, seed=2000 + rank)
    sd = torch.bfloat16 if cfg["dtype"] == "bf16" else torch.float32
    esz = 2 if cfg["dtype"] == "bf16" else 4
    t = lambda a, ty=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(ty)  # noqa: E731
    x, dt, A, B, C, D = t(v["x"], sd), t(v["dt"]), t(v["A"]), t(v["B"], sd), t(v["C"], sd), t(v["D"])
    state = t(v["state"])
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream(dev)

    def step():
        binding.step(state, x, dt, A, B, C, D=D, out=y)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    def max_ms(v):
        return max_over_ranks(v, world, dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_identity(local_rank)) as clk:
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = max_ms(e0.elapsed_time(e1))
    clocks = clk.summary()
    # end to end: each step copies the token's inputs in from pinned host memory
    # and reads y back (the state stays on the device, as in a generation loop)
    hx, hdt, hB, hC = (a.cpu().pin_memory() for a in (x, dt, B, C))
    hy = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    h2d = sum(a.numel() * a.element_size() for a in (hx, hdt, hB, hC))
    d2h = hy.numel() * hy.element_size()
    barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        x.copy_(hx, non_blocking=True)
        dt.copy_(hdt, non_blocking=True)
        B.copy_(hB, non_blocking=True)
        C.copy_(hC, non_blocking=True)
        step()
        hy.copy_(y, non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_ms(f0.elapsed_time(f1))
    if rank != 0:
        return
    bsz, H, P, N, G = cfg["batch"], cfg["nheads"], cfg["headdim"], cfg["dstate"], cfg["ngroups"]
    # algorithmic bytes of one step: the fp32 state read and written, x, y, dt, A, D, B, C
    step_bytes = 2 * bsz * H * P * N * 4 + 2 * bsz * H * P * esz + bsz * H * 4 + 2 * H * 4 + 2 * bsz * G * N * esz
    t_step = ms / args.steps * 1e-3
    peaks, peak_src = load_peaks()
    achieved = step_bytes / t_step / 1e9
    value = job_rate(world, bsz, args.steps, ms)
    line = {
        "metric": DECODE_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg["dtype"], "data": "synthetic",
        "config": {"workload": f"decode_2p7b: one token, B={bsz} H={H} P={P} N={N} G={G} {cfg['dtype']}, "
                               "fp32 state resident",
                   "batch": bsz, "nheads": H, "headdim": P, "dstate": N, "ngroups": G,
                   "l2": "no flush: the fp32 state exceeds L2 (126 MB)" if bsz * H * P * N * 4 > 126e6
                         else "no flush: the state fits in L2, so this line is L2-warm",
                   "parallelism": "replicas"},
        "roofline": {"bound": "hbm", "kernel": "ssd_step", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)"},
        "gpu_launches": args.steps,
        "e2e": {"value": job_rate(world, bsz, args.steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = decode_cpu_baseline(v)
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mamba2_2p7b", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--decode", action="store_true",
                    help="time the decode step (ssd_step) on its own shape instead of the scan")
    ap.add_argument("--backward", action="store_true",
                    help="time ssd_backward (the gradients of every input) on the workload")
    ap.add_argument("--block", action="store_true",
                    help="time ssd_forward_block: softplus(dt + dt_bias), the scan, y * silu(z) "
                         "and RMSNorm over each token's H * P values")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = dict(WORKLOADS[args.workload])
    cfg.setdefault("final_state", True)
    if args.block:
        cfg["block"] = True
    if args.batch is not None:
        cfg["batch"] = args.batch

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, cfg, rank)
        return
    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.decode:
            run_decode(args, rank, world, local_rank)
        elif args.backward:
            run_backward(args, cfg, rank, world, local_rank)
        else:
            run_gpu(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
