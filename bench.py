"""Benchmark: effective fwd+bwd TFLOP/s of block-/index-sparse attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole path over one batch of synthetic input resident in
HBM: tile lists from the block mask (or top-k indices), the forward (O, LSE) and the
backward (Delta, dQ/dK/dV, dQ cast).  The metric counts tensor-core work of ACTIVE
128x128 tiles only, per query head: forward 2*128*128*(Dqk+Dv) and backward
2*128*128*(3*Dqk+2*Dv) per tile (partial tiles count in full).  Rank 0 prints one
JSON line.  With N > 1 (torchrun) every rank runs the same workload on its own GPU
(independent replicas, weak scaling) and the time is the max over ranks.

`--impl reference` times the fp64 CPU oracle (the reference implementation of the
operation in this project) on a bounded sample of the same workload and prints the
same JSON line with "impl": "reference".
"""
import argparse
import ctypes
import datetime
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from index_sparse_attention_b200 import inputs as I  # noqa: E402

METRIC = "effective TFLOP/s fwd+bwd (active blocks only), % of B200 bf16 tensor peak"
DEFAULT_WORKLOAD = "long_causal_blocksparse_h16_s32768_d256"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def max_over_ranks(x, device):
    """Max of a per-rank float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(flop_per_rank_step, ms_per_step_max, world):
    """Whole-job TFLOP/s: the work of every rank divided by the slowest rank's step time."""
    return world * flop_per_rank_step / (ms_per_step_max * 1e-3) / 1e12


def peak_basis(peaks, clocks):
    """The bf16 peak a run is measured against: the burst figure (a cuBLAS GEMM timed
    alone) unless the run's own clock record shows power capping during the timed
    region, then the sustained figure (the same GEMM looped for seconds under the cap)."""
    capped = bool(clocks) and "sw_power_cap" in clocks.get("reasons", [])
    if capped:
        return float(peaks.get("bf16_tflops_sustained",
                               FALLBACK_PEAKS["bf16_tflops_sustained"])), "bf16_tflops_sustained"
    return float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])), "bf16_tflops"


def converter_bytes(w):
    """Algorithmic HBM bytes of one tile-list conversion: index mode reads the indices
    once, writes the presence bitmap and reads it back once (classification); both
    modes write the forward lists and read them back for the transposed ones."""
    Tm, Tn = -(-w.Sq // 128), -(-w.Sk // 128)
    lists = 4 * w.B * w.HK * (Tm * (Tn + 2) + Tn * (Tm + 2))
    if w.mode == "index":
        bitmap = 4 * w.B * w.HK * w.Sq * (-(-w.Sk // 32))
        return 4 * w.B * w.Sq * w.HK * w.topk + 2 * bitmap + 2 * lists
    return w.B * w.HK * (-(-w.Sq // w.bs)) * (-(-w.Sk // w.bs)) + 2 * lists


def tile_flops(w):
    """(forward, backward) tensor-core FLOP of one active 128x128 tile for one query head."""
    return 2 * 128 * 128 * (w.Dqk + w.Dv), 2 * 128 * 128 * (3 * w.Dqk + 2 * w.Dv)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return json.load(open(p)), "measured"
    return FALLBACK_PEAKS, "fallback"


def bwd_kernel_name(w, deterministic=False, form="auto", sms=148):
    """The backward main kernel that the library launches for this workload's head dims.
    At (192,128): one CTA per key tile ("whole") when chosen, or under "auto" when the
    grid of key tiles is at least twice the SM count; else (and in deterministic mode)
    the head-dim split over two CTAs (the rule of sparse_attn_set_backward_form)."""
    if (w.Dqk, w.Dv) == (256, 256):
        return "sparse_bwd_pair_kernel"
    if (w.Dqk, w.Dv) == (192, 128):
        tiles = -(-w.Sk // 128) * w.HK * w.B
        whole = not deterministic and (form == "whole" or (form == "auto" and tiles >= 2 * sms))
        return f"sparse_bwd_kernel<192,128,{1 if whole else 2}>"
    inst = {(64, 64): "128,128,1", (128, 128): "128,128,1"}
    return f"sparse_bwd_kernel<{inst.get((w.Dqk, w.Dv), '?')}>"


def source_code_sha(paths):
    """Hash of the code in `paths`: whole-line comments, blank lines and indentation are
    left out, so that a comment edit keeps a committed measurement of the code valid."""
    h = hashlib.sha256()
    for p in paths:
        with open(p, encoding="utf-8") as fh:
            for line in fh:
                t = line.strip()
                if t and not t.startswith("//"):
                    h.update(t.encode("utf-8") + b"\n")
    return h.hexdigest()[:16]


# the sources each backward main kernel is compiled from
BWD_SOURCES = {
    "sparse_bwd_pair_kernel": ("bwd_pair.cu", "sa_device.cuh", "det_order.cuh", "sa_kernels.h"),
    "sparse_bwd_kernel": ("bwd.cu", "sa_device.cuh", "det_order.cuh", "sa_kernels.h"),
}


def bwd_source_sha(kernel):
    files = BWD_SOURCES[kernel.split("<")[0]]
    return source_code_sha(os.path.join(ROOT, "index_sparse_attention_b200", "csrc", f)
                           for f in files)


def profiled_traffic(workload):
    """DRAM bytes per launch of the backward main kernel from a committed ncu summary,
    or None when absent or taken on a different kernel source."""
    p = os.path.join(ROOT, "profiles", "bwd_main_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("workload") != workload or d.get("source_sha") != bwd_source_sha(d["kernel"]):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi (read-only) while timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu, self.proc, self.lines = gpu_index, None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "20"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(self.NAMES, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "reasons": sorted(reasons), "samples": len(sm)}


# -----------------------------------------------------------------------------------
# CPU oracle: the cpu_baseline leg and the reference arm
# -----------------------------------------------------------------------------------
def active_tiles_per_row(w, inp):
    """Active key tiles of each (b, KV head, query tile), from the mask or indices."""
    Mt, Nt = -(-w.Sq // 128), -(-w.Sk // 128)
    if w.mode == "block":
        r = 128 // w.bs
        m = np.zeros((w.B, w.HK, Mt * r, Nt * r), np.uint8)
        m[:, :, :inp.mask.shape[2], :inp.mask.shape[3]] = inp.mask
        act = m.reshape(w.B, w.HK, Mt, r, Nt, r).max(axis=(3, 5))
        if w.causal:
            act = act * np.tril(np.ones((Mt, Nt), np.uint8))[None, None]
        return act.sum(-1)
    out = np.zeros((w.B, w.HK, Mt), np.int64)
    for b in range(w.B):
        for g in range(w.HK):
            for mt in range(Mt):
                rows = inp.idx[b, mt * 128:(mt + 1) * 128, g]
                ii = np.arange(mt * 128, mt * 128 + rows.shape[0])[:, None]
                ok = (rows >= 0) & ((rows <= ii) if w.causal else True)
                out[b, g, mt] = len(np.unique(rows[ok] // 128))
    return out


class OracleSampler:
    """Times the fp64 oracle on whole query tiles of the workload.

    Per sampled query tile (all 128 rows of one (b, h, m-tile)) the oracle computes the
    forward (O, LSE), Delta and the row side of the backward (recomputed S, dP, dS and
    dQ).  Work credited per active tile: 2*128*128*((Dqk+Dv) + (2*Dqk+Dv)) FLOP, i.e.
    the forward plus the S, dP and dQ contractions of the backward.
    """

    def __init__(self, w, inp, seed=0):
        import oracle
        self.oracle = oracle
        self.w, self.inp = w, inp
        self.P = oracle.Problem(inp.f32("q"), inp.f32("k"), inp.f32("v"), scale=w.scale,
                                causal=w.causal, mode=w.mode, mask=inp.mask, bs=w.bs, idx=inp.idx)
        self.do = inp.f32("do")
        self.act = active_tiles_per_row(w, inp)
        self.rng = np.random.default_rng(seed)
        self.per_tile = 2 * 128 * 128 * ((w.Dqk + w.Dv) + (2 * w.Dqk + w.Dv))
        self.cores = len(os.sched_getaffinity(0))

    def run_tile(self):
        w, o_ = self.w, self.oracle
        G = w.HQ // w.HK
        b, h = int(self.rng.integers(w.B)), int(self.rng.integers(w.HQ))
        mt = int(self.rng.integers(-(-w.Sq // 128)))
        i = np.arange(mt * 128, min(mt * 128 + 128, w.Sq))
        rows = np.stack([np.full(len(i), b), np.full(len(i), h), i], 1).astype(np.int64)
        o, lse = o_.forward_rows(self.P, rows)
        lse_full = np.zeros((w.B, w.HQ, w.Sq))
        dlt_full = np.zeros((w.B, w.HQ, w.Sq))
        lse_full[b, h, i] = lse
        dlt_full[b, h, i] = np.einsum("nd,nd->n", self.do[b, i, h].astype(np.float64), o)
        o_.backward_rows(self.P, self.do, lse_full, dlt_full, rows)
        return int(self.act[b, h // G, mt]) * self.per_tile

    def run_for(self, seconds, max_tiles=100000):
        flop, t0, n = 0, time.perf_counter(), 0
        while time.perf_counter() - t0 < seconds and n < max_tiles:
            flop += self.run_tile()
            n += 1
        return flop, time.perf_counter() - t0, n


def get_workload(args):
    w = I.WORKLOADS[args.workload]
    if args.seq:
        w = I.scaled(w, Sq=args.seq, Sk=args.seq, name=f"{w.name}@S{args.seq}")
    if getattr(args, "heads", ""):
        hq, hk = (int(x) for x in args.heads.split(","))
        if hq <= 0 or hk <= 0 or hq % hk:
            raise SystemExit("--heads wants HQ,HK with HQ a multiple of HK")
        w = I.scaled(w, HQ=hq, HK=hk, name=f"{w.name}@H{hq}x{hk}")
    return w


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:  # under torchrun only rank 0 runs the CPU reference
        return
    os.environ.setdefault("OMP_NUM_THREADS", str(len(os.sched_getaffinity(0))))
    w = get_workload(args)
    inp = I.make_inputs(w)
    s = OracleSampler(w, inp)
    per_step = args.ref_seconds or max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        s.run_for(per_step)
    flop, sec, tiles = 0, 0.0, 0
    for _ in range(args.steps):
        f, t, n = s.run_for(per_step)
        flop, sec, tiles = flop + f, sec + t, tiles + n
    value = flop / sec / 1e12
    sample = (f"{tiles} whole query tiles (128 rows of one (b, h, m-tile)) drawn at random over "
              f"{args.steps} steps of ~{per_step:.0f} s: fp64 forward + Delta + dQ-side backward "
              f"rows; credited 2*128^2*((Dqk+Dv)+(2*Dqk+Dv)) FLOP per active tile")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": int(args.gpus), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * sec / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, None),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": s.cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, active):
    cfg = {"workload": w.name, "B": w.B, "HQ": w.HQ, "HK": w.HK, "Sq": w.Sq, "Sk": w.Sk,
           "Dqk": w.Dqk, "Dv": w.Dv, "mode": w.mode, "causal": w.causal, "parallelism": "replicas"}
    if w.mode == "block":
        cfg.update(block=w.bs, density=w.density)
    else:
        cfg.update(topk=w.topk)
    if active is not None:
        cfg["active_tile_heads"] = active
    in_bytes = 2 * (w.B * w.Sq * w.HQ * (w.Dqk + w.Dv) + w.B * w.Sk * w.HK * (w.Dqk + w.Dv))
    cfg["l2"] = (f"inputs larger than L2: q, k, v, dO = {in_bytes / 2**20:.0f} MiB > 126 MiB"
                 if in_bytes > L2_BYTES else "L2 flushed between steps (256 MiB write)")
    return cfg


# -----------------------------------------------------------------------------------
# GPU arm
# -----------------------------------------------------------------------------------
def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))

    import index_sparse_attention_b200 as sa
    from index_sparse_attention_b200 import _lib

    L = _lib.load()
    sa.sparse_attn_set_forward_form(args.fwd_form)
    sa.sparse_attn_set_backward_form(args.bwd_form)
    w = get_workload(args)
    inp = I.make_inputs(w)
    dev = torch.device("cuda", local)

    def bf(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)

    host = {"q": bf(inp.q), "k": bf(inp.k), "v": bf(inp.v), "do": bf(inp.do)}
    if w.mode == "block":
        host["mask"] = torch.from_numpy(inp.mask)
    else:
        host["idx"] = torch.from_numpy(inp.idx)
    g = {k: v.to(dev) for k, v in host.items()}
    flush = None
    in_bytes = sum(t.numel() * t.element_size() for t in g.values())
    if in_bytes <= L2_BYTES:
        flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)

    def lists():
        if w.mode == "block":
            return sa.block_mask_to_block_sparse(g["mask"], w.B, w.HK, w.Sq, w.Sk, bs=w.bs,
                                                 causal=w.causal)
        return sa.index_to_block_sparse(g["idx"], w.Sk, causal=w.causal)

    ws = torch.empty(sa.sparse_attn_bwd_workspace_size(g["q"], g["k"], g["v"], lists()),
                     dtype=torch.uint8, device=dev)
    o = torch.empty((w.B, w.Sq, w.HQ, w.Dv), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.HQ, w.Sq), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(g["q"]), torch.empty_like(g["k"]), torch.empty_like(g["v"])

    def step(src=None):
        bsp = lists()
        sa.sparse_attn_fwd(g["q"], g["k"], g["v"], bsp, w.scale, o=o, lse=lse)
        sa.sparse_attn_bwd(g["q"], g["k"], g["v"], o, lse, g["do"], bsp, w.scale, dq=dq, dk=dk,
                           dv=dv, workspace=ws, deterministic=args.deterministic)
        return bsp

    bsp = step()
    torch.cuda.synchronize()
    active = bsp.active_tiles() * (w.HQ // w.HK)  # tile x query-head units
    fwd_f, bwd_f = tile_flops(w)
    flop_step = active * (fwd_f + bwd_f)

    for _ in range(args.warmup):
        step()
        if flush is not None:
            flush.zero_()
    torch.cuda.synchronize()

    # per-step events: 6 inside the library (fwd, bwd pre/main/post) + step bounds
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    stream = torch.cuda.current_stream(dev)
    for row in evs:
        for e in row:
            e.record(stream)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches_per_step = (3 if w.mode == "block" else 4) + 1 + 3 + (1 if flush is not None else 0)
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for s in range(args.steps):
            arr = (ctypes.c_void_p * 6)(*[ctypes.c_void_p(e.cuda_event) for e in evs[s]])
            L.sparse_attn_set_timing_events(arr)
            step()
            if flush is not None:
                flush.zero_()
        t_end.record(stream)
        torch.cuda.synchronize()
    L.sparse_attn_set_timing_events(None)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks(t_start.elapsed_time(t_end), dev)

    # the converter alone (it is part of every step above): mean over the same number of
    # calls, timed on the launch stream
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for _ in range(args.steps):
        lists()
    c1.record(stream)
    torch.cuda.synchronize()
    conv_ms = c0.elapsed_time(c1) / args.steps
    per_kernel = {
        "fwd": float(np.mean([r[0].elapsed_time(r[1]) for r in evs])),
        "bwd_pre": float(np.mean([r[2].elapsed_time(r[3]) for r in evs])),
        "bwd_main": float(np.mean([r[3].elapsed_time(r[4]) for r in evs])),
        "bwd_post": float(np.mean([r[4].elapsed_time(r[5]) for r in evs])),
    }
    ms_step = ms / args.steps
    value = whole_job_rate(flop_step, ms_step, world)

    # end to end through the public API with host buffers: every step copies its inputs
    # from pinned host memory and every output back.  As in a training loop that
    # prefetches, the copy of step s+1's inputs and the read-back of step s-1's outputs
    # run on their own streams while step s computes (device inputs and outputs
    # double-buffered; the events below order each buffer's reuse).
    pin = {k: v.pin_memory() for k, v in host.items()}
    outs = [[o, lse, dq, dk, dv], [torch.empty_like(t) for t in (o, lse, dq, dk, dv)]]
    gin = [g, {k: torch.empty_like(v) for k, v in g.items()}]
    pin_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs[0]]
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in outs[0])
    e_steps = max(1, min(args.steps, 10))
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def step_e2e(gs, os_):
        bsp = (sa.block_mask_to_block_sparse(gs["mask"], w.B, w.HK, w.Sq, w.Sk, bs=w.bs,
                                             causal=w.causal) if w.mode == "block"
               else sa.index_to_block_sparse(gs["idx"], w.Sk, causal=w.causal))
        sa.sparse_attn_fwd(gs["q"], gs["k"], gs["v"], bsp, w.scale, o=os_[0], lse=os_[1])
        sa.sparse_attn_bwd(gs["q"], gs["k"], gs["v"], os_[0], os_[1], gs["do"], bsp, w.scale,
                           dq=os_[2], dk=os_[3], dv=os_[4], workspace=ws,
                           deterministic=args.deterministic)

    def run_e2e(n):
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready, used, done, out_free = {}, {}, {}, {}
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_h2d.wait_event(e0)
        s_d2h.wait_event(e0)

        def load(i):
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(used[i - 2])
                for k in pin:
                    gin[i % 2][k].copy_(pin[k], non_blocking=True)
                in_ready[i] = ev()
                in_ready[i].record(s_h2d)

        load(0)
        for i in range(n):
            if i + 1 < n:
                load(i + 1)
            stream.wait_event(in_ready[i])
            if i >= 2:
                stream.wait_event(out_free[i - 2])
            step_e2e(gin[i % 2], outs[i % 2])
            used[i] = done[i] = ev()
            done[i].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(done[i])
                for src, dst in zip(outs[i % 2], pin_out):
                    dst.copy_(src, non_blocking=True)
                out_free[i] = ev()
                out_free[i].record(s_d2h)
        stream.wait_event(out_free[n - 1])
        stream.wait_event(in_ready[n - 1])
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    run_e2e(2)  # warm the copy streams and the second buffer set
    e_ms = max_over_ranks(run_e2e(e_steps), dev)
    e2e_value = whole_job_rate(flop_step, e_ms, world)

    peaks, peak_src = load_peaks()
    clocks = clk.summary()
    if rank == 0:
        peak, peak_kind = peak_basis(peaks, clocks)
        peak_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        peak_sust = float(peaks.get("bf16_tflops_sustained",
                                    FALLBACK_PEAKS["bf16_tflops_sustained"]))
        of = "of measured" if peak_src == "measured" else "of fallback"
        achieved = active * bwd_f / (per_kernel["bwd_main"] * 1e-3) / 1e12
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        conv_b = converter_bytes(w)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(workload_config(w, active),
                           **({"backward": "deterministic"} if args.deterministic else {}),
                           **({"forward_form": args.fwd_form} if args.fwd_form != "auto"
                              else {}),
                           **({"backward_form": args.bwd_form} if args.bwd_form != "auto"
                              else {})),
            "pct_of_bf16_peak": 100.0 * (value / world) / peak,
            "pct_basis": (f"{peak_kind} {peak:.1f} TFLOP/s ({of}); burst unless the clock record "
                          "of the timed region shows sw_power_cap"),
            "pct_of_bf16_burst": 100.0 * (value / world) / peak_burst,
            "pct_of_bf16_sustained": 100.0 * (value / world) / peak_sust,
            "flop_per_step": flop_step, "kernel_ms": per_kernel,
            "roofline": {
                "kernel": bwd_kernel_name(w, args.deterministic, args.bwd_form,
                                          torch.cuda.get_device_properties(dev).multi_processor_count),
                "bound": "tensor",
                "achieved": achieved,
                "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_kind": f"{peak_kind} ({of}); burst {peak_burst:.1f}, sustained {peak_sust:.1f}",
                "traffic": profiled_traffic(w.name),
                "algorithmic": "2*128*128*(3*Dqk+2*Dv) FLOP per active tile x query head",
            },
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e_ms, "steps": e_steps,
                    "overlap": "H2D of step s+1 and D2H of step s-1 on their own streams "
                               "while step s computes; device inputs and outputs "
                               "double-buffered"},
            "converter": {
                "ms": conv_ms, "algorithmic_bytes": conv_b, "achieved_gbs": conv_b / conv_ms / 1e6,
                "peak_gbs": hbm, "frac": conv_b / conv_ms / 1e6 / hbm,
                "kernels": ("scatter_bits + classify_index + compact + transpose" if w.mode == "index"
                            else "classify_block + compact + transpose"),
                "note": "timed alone, same launches as inside each step"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            os.environ.setdefault("OMP_NUM_THREADS", str(len(os.sched_getaffinity(0))))
            s = OracleSampler(w, inp)
            s.run_tile()  # load and warm the library
            f, sec, n = s.run_for(args.cpu_seconds)
            line["cpu_baseline"] = {
                "value": f / sec / 1e12, "unit": "TFLOP/s", "cores": s.cores, "kind": "oracle",
                "sample": (f"{n} random whole query tiles of the workload, {sec:.1f} s: fp64 "
                           "forward + Delta + dQ-side backward rows; credited "
                           "2*128^2*((Dqk+Dv)+(2*Dqk+Dv)) FLOP per active tile")}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# -----------------------------------------------------------------------------------
# Top-k selector (the producer of index mode's indices), measured on its own
# -----------------------------------------------------------------------------------
TOPK_METRIC = "top-k selector time per packed sequence (ms)"
# the pages' standalone medians of their TileLang selector (hardware not stated), per
# pack length: context only
TOPK_PAGE_MS = {16384: 2.660752, 32768: 5.570000, 65536: 12.461776, 131072: 30.375248}


def run_gather(args):
    """Token-gather forward (sparse_attn_fwd_gather) against the block forward on an index
    workload: both timed with CUDA events on the same inputs, and the gather path's
    volume (the K/V rows it gathers) and token-level rate."""
    import torch

    import index_sparse_attention_b200 as sa

    w = get_workload(args)
    if w.mode != "index":
        raise SystemExit("--op gather needs an index workload")
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    inp = I.make_inputs(w, with_grad=False)

    def bf(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v = bf(inp.q), bf(inp.k), bf(inp.v)
    idx = torch.from_numpy(inp.idx).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    bsp = sa.index_to_block_sparse(idx, w.Sk, causal=w.causal, dev_status=status)
    o = torch.empty((w.B, w.Sq, w.HQ, w.Dv), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.HQ, w.Sq), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    with ClockSampler(dev.index) as clk:
        g_ms = timed(lambda: sa.sparse_attn_fwd_gather(q, k, v, bsp, w.scale, o=o, lse=lse,
                                                       dev_status=status))
        b_ms = timed(lambda: sa.sparse_attn_fwd(q, k, v, bsp, w.scale, o=o, lse=lse,
                                                dev_status=status))
    assert int(status.item()) == 0
    # selected (query, KV head) keys: distinct entries below the causal limit
    pairs = 0
    qpos = np.arange(w.Sq)[None, :, None, None]
    for b in range(w.B):
        x = np.sort(inp.idx[b:b + 1], axis=-1)
        ok = x >= 0
        if w.causal:
            ok &= x <= qpos
        ok[..., 1:] &= x[..., 1:] != x[..., :-1]
        pairs += int(ok.sum())
    G = w.HQ // w.HK
    gathered = pairs * (w.Dqk + w.Dv) * 2
    token_flop = pairs * G * 2 * (w.Dqk + w.Dv)
    active = int(bsp.cnt.reshape(-1, 2).sum())
    block_flop = active * w.HQ // w.HK * 2 * 128 * 128 * (w.Dqk + w.Dv)
    print(json.dumps({
        "op": "gather_vs_block_forward", "workload": w.name, "steps": args.steps,
        "warmup": args.warmup, "gather_ms": g_ms, "block_ms": b_ms, "gather_over_block": g_ms / b_ms,
        "gathered_bytes": gathered, "gather_gbs": gathered / (g_ms * 1e-3) / 1e9,
        "token_level_tflop": token_flop / 1e12,
        "token_level_tflops_gather": token_flop / (g_ms * 1e-3) / 1e12,
        "block_counted_tflop": block_flop / 1e12,
        "block_tflops_block_path": block_flop / (b_ms * 1e-3) / 1e12,
        "token_level_tflops_block_path": token_flop / (b_ms * 1e-3) / 1e12,
        "clocks": clk.summary(), "data": "synthetic",
    }))


def run_topk(args):
    import torch

    import index_sparse_attention_b200 as sa
    from index_sparse_attention_b200 import _lib

    L = _lib.load()
    n, k = args.pack, args.k
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    host = I.topk_scores(n, n, seed=6000)
    starts, ends = I.packed_causal_ranges(n)
    scores = torch.from_numpy(host).to(dev)
    st, en = torch.from_numpy(starts).to(dev), torch.from_numpy(ends).to(dev)
    idx = torch.empty((n, k), dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(args.warmup):
        sa.topk_select(scores, k, st, en, out_idx=idx, dev_status=status)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            sa.topk_select(scores, k, st, en, out_idx=idx, dev_status=status)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    assert int(status.item()) == 0
    # end to end: pinned scores in, indices out, every step
    pin_s = torch.from_numpy(host).pin_memory()
    pin_i = torch.empty((n, k), dtype=torch.int32, pin_memory=True)
    e_steps = max(1, min(args.steps, 5))
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e_steps):
        scores.copy_(pin_s, non_blocking=True)
        sa.topk_select(scores, k, st, en, out_idx=idx, dev_status=status)
        pin_i.copy_(idx, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1) / e_steps
    peaks, src = load_peaks()
    read_bytes = 4 * int((ends.astype(np.int64) - starts).sum())
    bytes_step = read_bytes + 4 * n * k
    achieved = bytes_step / (ms * 1e-3) / 1e9
    line = {
        "metric": TOPK_METRIC, "value": ms, "unit": "ms", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"topk_pack{n}_k{k}", "rows": n, "cols": n, "k": k,
                   "ranges": "one packed causal segment: row i selects from [0, i+1)",
                   "scores": "standard normal fp32 (seed 6000)",
                   "l2": f"inputs larger than L2: scores {4 * n * n / 2**20:.0f} MiB"},
        "pages_context_ms": TOPK_PAGE_MS.get(n),
        "roofline": {"kernel": "topk_kernel", "bound": "hbm", "achieved": achieved,
                     "peak": float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])), "unit": "GB/s",
                     "frac": achieved / float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])),
                     "traffic": None,
                     "algorithmic": "4 B per valid score read once + 4 B per output index"},
        "e2e": {"value": e_ms, "unit": "ms", "h2d_bytes_per_step": 4 * n * n,
                "d2h_bytes_per_step": 4 * n * k},
        "gpu_launches": args.steps, "clocks": clk.summary(),
    }
    if not args.no_cpu_baseline:
        from oracle import topk as T
        rng = np.random.default_rng(0)
        t0, rows_done, work = time.perf_counter(), 0, 0
        while time.perf_counter() - t0 < args.cpu_seconds:
            r = int(rng.integers(n))
            T.topk_select(host, k, starts, ends, rows=[r])
            rows_done += 1
            work += int(ends[r] - starts[r])
        sec = time.perf_counter() - t0
        total = int((ends.astype(np.int64) - starts).sum())
        line["cpu_baseline"] = {
            "value": 1e3 * sec * total / max(1, work), "unit": "ms", "cores": 1, "kind": "oracle",
            "sample": f"{rows_done} random rows ({work} valid scores) in {sec:.1f} s, one numpy sort "
                      "per row, scaled to the whole pack by its number of valid scores"}
    print(json.dumps(line), flush=True)


# -----------------------------------------------------------------------------------
# Index-workload statistics (CPU): what finer-grained or gathering designs could skip
# -----------------------------------------------------------------------------------
def run_index_stats(args):
    """Counts on the seeded index workload, per KV head, from the indices alone:
    - active 128 x 128 tiles (the block path's unit) and their block-counted FLOP against
      the token-level FLOP of the selected (query, key) pairs;
    - among the 128-query x 32-key sub-blocks of active tiles, the share holding at least
      one selected pair (a kernel that skipped empty 32-key sub-blocks could save the rest);
    - per 128-query tile, the union of its rows' key sets against the tile's causal key
      range (what a kernel gathering that union for the whole tile would still do);
    - the K/V rows a per-(token, KV head) gather would move per forward, and how many
      query heads share each gathered row (its reuse)."""
    w = I.WORKLOADS[args.workload]
    if w.mode != "index":
        raise SystemExit("--op index_stats needs an index workload")
    if args.seq:
        w = I.scaled(w, Sq=args.seq, Sk=args.seq, name=f"{w.name}@S{args.seq}")
    t0 = time.perf_counter()
    idx = I.topk_indices(w)
    G = w.HQ // w.HK
    Tm, Tn = -(-w.Sq // 128), -(-w.Sk // 128)
    sel = tiles = sub_nonempty = sub_total = 0
    union_keys = range_keys = 0
    for b in range(w.B):
        for g in range(w.HK):
            present = np.zeros((w.Sq, Tn * 128), dtype=bool)
            rows = np.repeat(np.arange(w.Sq), w.topk)
            keys = idx[b, :, g, :].reshape(-1)
            ok = keys >= 0
            if w.causal:
                ok &= keys <= rows
            present[rows[ok], keys[ok]] = True
            sel += int(present.sum())
            pad = np.zeros((Tm * 128, Tn * 128), dtype=bool)
            pad[:w.Sq] = present
            sub = pad.reshape(Tm, 128, Tn * 4, 32).any(axis=(1, 3))  # [Tm, Tn*4]
            act = sub.reshape(Tm, Tn, 4).any(axis=2)                   # [Tm, Tn]
            tiles += int(act.sum())
            sub_total += int(act.sum()) * 4
            sub_nonempty += int(sub.reshape(Tm, Tn, 4)[act].sum())
            union = pad.reshape(Tm, 128, Tn * 128).any(axis=1)        # [Tm, keys]
            union_keys += int(union.sum())
            for mt in range(Tm):
                hi = min((mt + 1) * 128, w.Sk) if w.causal else w.Sk
                range_keys += hi
    flop_block = tiles * G * 2 * 128 * 128 * (w.Dqk + w.Dv)
    flop_token = sel * G * 2 * (w.Dqk + w.Dv)
    gather_bytes = sel * 2 * (w.Dqk + w.Dv)  # one K and one V row per selected pair
    line = {
        "op": "index_stats", "workload": w.name, "seconds": time.perf_counter() - t0,
        "selected_pairs_per_kv_head": sel / (w.B * w.HK),
        "active_tiles": tiles, "forward_flop_block_counted": flop_block,
        "forward_flop_token_level": flop_token,
        "block_over_token": flop_block / max(1, flop_token),
        "nonempty_32key_subblocks_of_active_tiles": sub_nonempty / max(1, sub_total),
        "tile_union_keys_over_causal_range": union_keys / max(1, range_keys),
        "token_gather_forward_bytes": gather_bytes,
        "token_gather_row_reuse_query_heads": G,
        "block_path_forward_bytes_per_tile_visit": 128 * 2 * (w.Dqk + w.Dv),
        "block_path_row_reuse_query_heads": 128 * G,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(I.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=0.0,
                    help="CPU seconds per reference step (default: the run ends in ~2.5 min)")
    ap.add_argument("--seq", type=int, default=0,
                    help="override Sq = Sk (smaller profiling captures of the same kernels)")
    ap.add_argument("--deterministic", action="store_true",
                    help="use the deterministic backward (fixed-order dQ accumulation)")
    ap.add_argument("--heads", default="",
                    help="override the head counts as HQ,HK (e.g. 16,8: GQA on the D=256 workload)")
    ap.add_argument("--fwd-form", default="auto",
                    choices=["auto", "one_head", "cta_pair", "two_heads", "two_tiles"],
                    help="forward form: one CTA per query tile and head, two heads of a "
                         "GQA group on a 2-CTA pair with cta_group::2 MMAs, two heads per "
                         "CTA, two query tiles of one head per CTA, or the library's choice "
                         "(auto)")
    ap.add_argument("--bwd-form", default="auto", choices=["auto", "split", "whole"],
                    help="backward form at head dims (192,128): two CTAs per key tile each "
                         "with part of the head dim, one CTA per key tile, or the library's "
                         "choice by grid size (auto)")
    ap.add_argument("--op", default="attention",
                    choices=["attention", "topk", "index_stats", "gather"],
                    help="topk: time the top-k selector alone on one packed sequence; "
                         "index_stats: counts on an index workload (CPU only); gather: the "
                         "token-gather forward against the block forward (index workload)")
    ap.add_argument("--pack", type=int, default=16384, help="--op topk: packed sequence length")
    ap.add_argument("--k", type=int, default=2048, help="--op topk: k")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.op == "topk":
        run_topk(args)
        return
    if args.op == "index_stats":
        run_index_stats(args)
        return
    if args.op == "gather":
        run_gather(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
