"""Benchmark of SGMV expand-slice on B200.

One step = the whole hot path over one batch: the three expand-slice calls of a
Llama-7B fused-QKV prefill batch (16 sequences with lengths uniform in
[64, 1024], rank 16, 32 adapters with 10% of sequences at -1, bf16, slices of
4096 at offsets 0/4096/8192 of a T x 12288 output, add_inputs=True).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--variant auto|simt|tc]

Timing: inputs are resident in HBM; W untimed warm-up steps; then K steps as
CUDA-graph replays (each graph holds up to 100 steps of back-to-back kernel
launches), timed by CUDA events on the launching stream around the whole
region and bracketed by a barrier and a device synchronise on both sides; max
over ranks.  The kernel's average launch duration is the region time divided
by the launches in it (kernels run back to back; gaps between them count).  The output (215 MB
for the default workload) is larger than L2 and every step streams all of it,
so no flush is needed between steps; `l2_flushed` reports the median of 60
steps with a 256 MiB write before each, to show it.  `eager` times 100 steps
of plain calls without a graph and the host time inside each call.  `value`
is algorithmic HBM bytes of all ranks / time; `configs` holds the same
figures for each of the five expand-slice workloads (their own inputs);
`e2e` repeats the measurement through the same C-ABI calls with the inputs in
pinned host memory, copying them in and the output back every step.
`--impl reference` times the CPU oracle on host cores instead (rank 0).
"""
import argparse
import ctypes
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import sgmv_inputs as gen  # noqa: E402

METRIC = "sgmv_expand_slice achieved HBM GB/s (% of B200 roofline) and tokens/s per call"
FALLBACK_HBM_GBS = 6650.0
STEPS_PER_GRAPH = 100
L2_BYTES = 126 << 20            # B200 L2
MAX_COPIES = 8                  # most input copies a workload rotates through

WORKLOAD_TEXT = {
    "qkv_prefill": "Llama-7B fused-QKV prefill: 16 seqs U[64,1024], rank 16, 32 adapters (10% idx -1), "
                   "bf16, 3 slices of 4096 into T x 12288, add_inputs",
    "mlp_mixed": "MLP gate/up: 64 seqs Geom(mean 256)<=2048, rank 64, fp32 x vs bf16 4-D weights "
                 "(128 adapters), bf16 out T x 22016, 2 slices of 11008, add_inputs",
    "long_single": "single-tenant long prefill: 1 x 32768 tokens, rank 8, fp16, 4096 slice, overwrite",
    "decode_mix": "decode-like mix: 256 seqs Zipf(1.2) in [1,64], rank 32, 256 distinct adapters "
                  "(10% -1), bf16, slice 5120 at 5120 of T x 15360, add_inputs",
    "tiny": "tiny: 4 seqs [4,6,3,7], rank 16, fp16, slice 128 at 128, overwrite",
    "decode_bgmv": "decode step (bgmv_expand_slice): 256 one-token rows, 256 distinct adapters (10% -1), "
                   "rank 32, bf16, slice 5120 at 5120 of 256 x 15360, add_inputs",
    "qkv_shrink": "LoRA-A shrink feeding the QKV prefill (sgmv_shrink): 16 seqs U[64,1024], 32 adapters "
                  "(10% -1), hidden 4096 -> rank 16, bf16, split-H workspace",
}

DT_SIZE = {"f16": 2, "bf16": 2, "f32": 4}

# the five expand-slice workloads every default run reports (the `configs` key)
CONFIG_WORKLOADS = ("tiny", "qkv_prefill", "mlp_mixed", "long_single", "decode_mix")


# ---------------------------------------------------------------- accounting

def call_accounting(p: gen.Problem, call: int):
    """Algorithmic bytes and flops of one expand-slice call, from the metadata."""
    c = p.calls[call]
    A, N, K = c.w.shape[0], c.slice_size, p.rank
    ok = (p.lora_idx >= 0) & (p.lora_idx < A) & (p.seq_len > 0) & (p.seq_start >= 0)
    rows = int(p.seq_len[ok].sum())
    adapters = len(np.unique(p.lora_idx[ok]))
    meta = (1 if p.op == "bgmv" else 3) * p.batches * (8 if p.meta_dt == "int64" else 4)
    sx, sw, so = DT_SIZE[p.x_dt], DT_SIZE[p.w_dt], DT_SIZE[p.out_dt]
    byts = rows * (K * sx + N * so * (2 if p.add_inputs else 1)) + adapters * N * K * sw + meta
    flops = 2 * N * K * rows
    return byts, flops, rows


def step_accounting(p):
    b = f = r = 0
    for c in range(len(p.calls)):
        bb, ff, rr = call_accounting(p, c)
        b, f, r = b + bb, f + ff, r + rr
    return b, f, r


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the source files each kernel family is compiled from (its own header, the PTX
# wrappers and the shared helpers); a recorded DRAM figure stays valid while their
# code (comments and layout aside) is unchanged
KERNEL_SOURCES = {
    "tc": ("common.cuh", "tc.cuh", "tc_kernel.cuh", "tc_ptx.cuh"),
    "simt": ("common.cuh", "simt.cuh"),
    "decode": ("common.cuh", "bgmv.cuh"),
    "shrink": ("common.cuh", "tc_ptx.cuh", "shrink.cuh"),
}


_COMMENTS = re.compile(r"//[^\n]*|/\*.*?\*/", re.S)


def code_only(text):
    """C++ source without comments, whitespace runs collapsed."""
    return " ".join(_COMMENTS.sub(" ", text).split())


def kernel_source_hash(variant):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "segmented_gather_gemm_expand_b200", "csrc")
    for fn in KERNEL_SOURCES[variant]:
        h.update(fn.encode())
        h.update(code_only(open(os.path.join(csrc, fn), encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def _traffic_entry(workload, variant):
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(path))
        e = d[workload][variant]
        if e.get("kernel_source_hash") == kernel_source_hash(variant):
            return e
    except Exception:
        pass
    return None


def recorded_traffic(workload, variant):
    """DRAM bytes (read + write) per launch from a committed ncu summary, if taken on the current kernel source."""
    e = _traffic_entry(workload, variant)
    return float(e["dram_read_bytes_per_launch"] + e["dram_write_bytes_per_launch"]) if e else None


def recorded_traffic_split(workload, variant):
    e = _traffic_entry(workload, variant)
    if not e:
        return None
    rd, wr = float(e["dram_read_bytes_per_launch"]), float(e["dram_write_bytes_per_launch"])
    return {"traffic": rd + wr, "read": rd, "write": wr}


# ---------------------------------------------------------------- ranks

def reduce_over_ranks(total_ms, step_bytes, step_flops, tokens, device, world):
    """Whole-job figures: the slowest rank's time, the sum of every rank's work.
    Each rank runs its own batch (no data-path collective); this is the only
    communication, outside the timed region."""
    if world == 1:
        return float(total_ms), float(step_bytes), float(step_flops), float(tokens)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(total_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    w = torch.tensor([float(step_bytes), float(step_flops), float(tokens)], dtype=torch.float64, device=device)
    dist.all_reduce(w)
    b, f, n = (float(v) for v in w.tolist())
    return float(t.item()), b, f, n


# ---------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.bus_id = (bus_id or "").lower()
        self.proc = None
        self.path = os.path.join("/tmp", f"sgmv_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            if self.bus_id and self.bus_id not in parts[1].lower():
                continue
            rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[6:10]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][3]) if rows[0][3].replace(".", "").isdigit() else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------- runtime helpers

def make_calls(p, dev_tensors, sg_abi, stream_handle_fn, workspace=None):
    """Pre-marshalled C-ABI argument tuples, one per slice call."""
    import segmented_gather_gemm_expand_b200 as sg
    x, ws, y, meta = dev_tensors
    wsp = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else None
    wsb = workspace.numel() if workspace is not None else 0
    descs = []
    for c, call in enumerate(p.calls):
        d = [sg._desc(t) for t in (x, ws[c], y, *meta)]
        descs.append((d, call.slice_offset, call.slice_size))
    lib = sg._lib

    def run(c, stream):
        d, off, size = descs[c]
        if p.op == "shrink":
            rc = lib.sgmv_shrink(*[ctypes.byref(t) for t in d], p.batches, p.max_seq_len, wsp, wsb,
                                 ctypes.c_void_p(stream))
        elif p.op == "bgmv":   # x, B, out and lora_idx only: row b is one token
            rc = lib.bgmv_expand_slice(ctypes.byref(d[0]), ctypes.byref(d[1]), ctypes.byref(d[2]),
                                       ctypes.byref(d[5]), p.batches, off, size, int(p.add_inputs),
                                       ctypes.c_void_p(stream))
        else:
            rc = lib.sgmv_expand_slice(*[ctypes.byref(t) for t in d], p.batches, p.max_seq_len, off, size,
                                       int(p.add_inputs), ctypes.c_void_p(stream))
        if rc != 0:
            raise sg.SgmvError(rc, {"bgmv": "bgmv_expand_slice", "shrink": "sgmv_shrink"}.get(p.op, "sgmv_expand_slice"))
    return run, descs


def make_multi_call(p, dev_tensors):
    """Pre-marshalled arguments of ONE multi-slice call covering every slice."""
    import segmented_gather_gemm_expand_b200 as sg
    x, ws, y, meta = dev_tensors
    xd, yd = sg._desc(x), sg._desc(y)
    md = [sg._desc(t) for t in meta]
    wd = [sg._desc(w) for w in ws]
    n = len(wd)
    arr = (ctypes.POINTER(sg._abi.SgmvTensor) * n)(*[ctypes.pointer(w) for w in wd])
    offs = (ctypes.c_int64 * n)(*[c.slice_offset for c in p.calls])
    keep = (xd, yd, md, wd, arr, offs)
    lib = sg._lib

    def run(stream):
        rc = lib.sgmv_expand_multi_slice(ctypes.byref(xd), arr, n, ctypes.byref(yd),
                                         *[ctypes.byref(t) for t in md], p.batches, p.max_seq_len, offs,
                                         int(p.add_inputs), ctypes.c_void_p(stream))
        if rc != 0:
            raise sg.SgmvError(rc, "sgmv_expand_multi_slice")
    run.keep = keep
    return run


def graph_chunk(period):
    """Steps per captured graph: at most STEPS_PER_GRAPH, a multiple of the
    input rotation's period so that every replay continues the rotation."""
    return max(period, STEPS_PER_GRAPH // period * period)


def time_graph_region(step, steps, stream, torch, period=1):
    """Capture `steps` calls of step(stream_handle) as graphs of <= STEPS_PER_GRAPH
    steps, replay them once untimed, then time one replay of all of them with
    CUDA events on `stream`.  Returns milliseconds."""
    graphs = []
    remaining = steps
    while remaining > 0:
        s = min(graph_chunk(period), remaining)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            cs = torch.cuda.current_stream().cuda_stream
            for _ in range(s):
                step(cs)
        graphs.append(g)
        remaining -= s
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for g in graphs:
            g.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    del graphs
    return ms


# ---------------------------------------------------------------- our arm

SECONDARY_STEPS = 200        # graph-replayed steps for each extra config (at least)
FLUSH_BYTES = 256 << 20      # the L2 flush between steps of the flushed timing
FLUSH_STEPS = 60             # steps of the flushed timing (median reported)
EAGER_STEPS = 100            # steps of the eager (no graph) timing


def footprint_bytes(p):
    """Device bytes of a workload's buffers: x, the weights, the output and the metadata."""
    return int(p.x.base.nbytes if p.x.base is not None else p.x.nbytes) + sum(int(c.w.nbytes) for c in p.calls) \
        + int(p.y0.nbytes) + 3 * 8 * len(p.seq_start)


def l2_copies(p):
    """Copies of the workload's device buffers that the timed steps rotate through.

    1 when one copy is larger than L2 (every step streams it from HBM anyway);
    otherwise enough copies that the others, touched between two uses of one,
    exceed L2, so that each step reads its inputs from HBM; at most MAX_COPIES.
    Returns (copies, enough)."""
    f = max(footprint_bytes(p), 1)
    if f > L2_BYTES:
        return 1, True
    k = -(-L2_BYTES // f) + 1
    return min(k, MAX_COPIES), k <= MAX_COPIES


def l2_text(p):
    k, enough = l2_copies(p)
    mb = footprint_bytes(p) / 1e6
    if k == 1:
        return (f"no flush between steps: the step's buffers ({mb:.0f} MB) are larger than L2 and every step "
                f"streams its output (a flushed median is reported beside it)")
    if enough:
        return (f"{k} copies of the inputs ({mb:.0f} MB each) used in turn: the {(k - 1) * mb:.0f} MB of the other "
                f"copies touched between two uses of one exceed L2, so each step reads its inputs from HBM")
    return (f"inputs of {mb:.2f} MB: {k} copies used in turn still fit in L2, so this is not an HBM-bound "
            f"figure")


def workload_config(p, name, world, step_fused=False):
    """The `config` object of a bench line: the workload, identical in both arms."""
    _, _, rows = step_accounting(p)
    ncalls = len(p.calls)
    return {"workload": WORKLOAD_TEXT[name], "name": name,
            "batches": p.batches, "tokens_per_rank": p.total_tokens,
            "active_tokens_per_rank": rows // max(ncalls, 1), "rank": p.rank,
            "slices": ncalls, "slice_size": p.calls[0].slice_size,
            "adapters": int(p.calls[0].w.shape[0]), "add_inputs": bool(p.add_inputs),
            "x_dtype": p.x_dt, "w_dtype": p.w_dt, "out_dtype": p.out_dt,
            "parallelism": f"replicas x{world} (independent batches, no collective)",
            "l2": l2_text(p),
            "seed": p.seed,
            "step": ("all slices in one sgmv_expand_multi_slice call" if step_fused else
                     f"{ncalls} separate call(s)")}


class Resident:
    """A workload's inputs resident in HBM, with its C-ABI calls pre-marshalled.

    With copies > 1 the device buffers exist that many times and step() uses
    them in turn (see l2_copies); r.x, r.ws, r.y and r.meta are the first copy."""

    def __init__(self, p, device, copies=1):
        import torch
        import segmented_gather_gemm_expand_b200 as sg
        self.p = p
        tdt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}

        def host_tensor(a, dt):
            t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if dt != "f32" else np.ascontiguousarray(a))
            return t.view(tdt[dt]) if dt != "f32" else t

        self.hx = host_tensor(p.x, p.x_dt)
        self.hws = [host_tensor(c.w, p.w_dt) for c in p.calls]
        self.hy = host_tensor(p.y0, p.out_dt)
        self.hmeta = [torch.from_numpy(a.astype(np.int64)) for a in (p.seq_start, p.seq_len, p.lora_idx)]
        self.x = self.hx.to(device)
        self.ws = [w.to(device) for w in self.hws]
        self.y = self.hy.to(device)
        self.meta = [m.to(device) for m in self.hmeta]
        self.workspace = None
        x, ws, y, meta = self.x, self.ws, self.y, self.meta
        if p.op == "shrink":
            _, _, pref = sg.shrink_plan(x, ws[0], y, *meta, p.batches, p.max_seq_len, 1 << 34)
            self.workspace = torch.empty(max(pref, 16), dtype=torch.uint8, device=device)
        self.run, _ = make_calls(p, (x, ws, y, meta), None, None, workspace=self.workspace)
        self.period = max(1, copies)
        self.runs = [self.run]
        self._copies = []
        for _ in range(1, self.period):
            cx, cws, cy = x.clone(), [w.clone() for w in ws], y.clone()
            cmeta = [m.clone() for m in meta]
            cwsp = torch.empty_like(self.workspace) if self.workspace is not None else None
            self._copies.append((cx, cws, cy, cmeta, cwsp))
            self.runs.append(make_calls(p, (cx, cws, cy, cmeta), None, None, workspace=cwsp)[0])
        self.turn = 0
        self.ncalls = len(p.calls)
        self.shrink_splits = 0
        if p.op == "shrink":
            v_used, self.shrink_splits, _ = sg.shrink_plan(x, ws[0], y, *meta, p.batches, p.max_seq_len,
                                                           self.workspace.numel())
        elif p.op == "bgmv":
            v_used = sg.bgmv_plan(x, ws[0], y, meta[2], p.calls[0].slice_offset, p.calls[0].slice_size,
                                  p.add_inputs)
        else:
            v_used = sg.plan(x, ws[0], y, *meta, p.batches, p.max_seq_len, p.calls[0].slice_offset,
                             p.calls[0].slice_size, p.add_inputs)
        self.variant = {1: "simt", 2: "tc", 3: "decode"}.get(v_used, str(v_used))
        # which kernel family's source a recorded DRAM figure must match
        self.kernel_family = "shrink" if (p.op == "shrink" and self.variant == "tc") else self.variant
        # kernel launches one call makes (a split shrink adds the partial-sum reduction)
        self.launches_per_call = 2 if (p.op == "shrink" and self.shrink_splits > 1) else 1

    def step(self, st):
        """One step on the next copy of the buffers."""
        run = self.runs[self.turn]
        self.turn = (self.turn + 1) % self.period
        for c in range(self.ncalls):
            run(c, st)

    def step_first_copy(self, st):
        for c in range(self.ncalls):
            self.run(c, st)

    def multi_call(self):
        return make_multi_call(self.p, (self.x, self.ws, self.y, self.meta))


def warm(step, n, stream, torch):
    with torch.cuda.stream(stream):
        for _ in range(n):
            step(stream.cuda_stream)
    torch.cuda.synchronize()


def time_flushed(step, steps, stream, torch, device):
    """Per-step device time with a FLUSH_BYTES write (larger than L2) before every step;
    events bracket the step alone.  Returns the list of per-step milliseconds."""
    buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(steps):
            buf.fill_(i & 0xFF)
            ev[i][0].record(stream)
            step(stream.cuda_stream)
            ev[i][1].record(stream)
    torch.cuda.synchronize()
    out = [a.elapsed_time(b) for a, b in ev]
    del buf
    return out


def time_eager(step, steps, stream, torch):
    """Back-to-back eager calls (no graph): device time of the region, and host
    time spent inside the calls (argument checks, planning, tensor maps, launch)."""
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t0.record(stream)
        h0 = time.perf_counter()
        for _ in range(steps):
            step(stream.cuda_stream)
        h1 = time.perf_counter()
        t1.record(stream)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1), (h1 - h0) * 1e3


def secondary_entry(name, seed, steps, warmup, device, peak):
    """Graph-timed figures of one more workload (its own inputs, freed afterwards)."""
    import torch
    import segmented_gather_gemm_expand_b200 as sg
    p = gen.WORKLOADS[name](seed=seed)
    r = Resident(p, device, copies=l2_copies(p)[0])
    stream = torch.cuda.Stream(device)
    warm(r.step, warmup, stream, torch)
    steps = -(-steps // r.period) * r.period
    ms = time_graph_region(r.step, steps, stream, torch, r.period)
    assert sg.device_error(device) == 0, "a kernel reported a device-side error"
    b, f, rows = step_accounting(p)
    ncalls = r.ncalls
    us_call = ms * 1e3 / (steps * ncalls)
    call_bytes = b / ncalls
    entry = {"workload": WORKLOAD_TEXT[name], "variant": r.variant, "calls_per_step": ncalls,
             "us_per_call": us_call, "gb_s": call_bytes / (us_call * 1e-6) / 1e9,
             "frac": call_bytes / (us_call * 1e-6) / 1e9 / peak,
             "tokens_per_s": p.total_tokens * steps / (ms * 1e-3),
             "tflops": f * steps / (ms * 1e-3) / 1e12, "bytes_per_call": call_bytes, "steps": steps,
             "traffic": recorded_traffic(name, r.kernel_family), "l2": l2_text(p)}
    del r
    torch.cuda.empty_cache()
    return entry


def bench_ours(args, rank, world, device):
    import torch
    import segmented_gather_gemm_expand_b200 as sg

    torch.cuda.set_device(device)
    variants = {"auto": sg.VARIANT_AUTO, "simt": sg.VARIANT_SIMT, "tc": sg.VARIANT_TC}
    sg.set_variant(variants[args.variant])
    p = gen.WORKLOADS[args.workload](seed=args.seed + rank)
    r = Resident(p, device, copies=1 if args.step == "fused" else l2_copies(p)[0])
    ncalls = r.ncalls
    # One step: the slice calls one by one, or (--step fused) all slices in one
    # sgmv_expand_multi_slice call.
    fused_step = args.step == "fused" and ncalls > 1 and p.op == "slice"
    if fused_step:
        run_multi_step = r.multi_call()
        _, launches_per_step = sg.plan_multi_slice(r.x, r.ws, r.y, *r.meta, p.batches, p.max_seq_len,
                                                   [c.slice_offset for c in p.calls], p.add_inputs)

        def step_fn(st):
            run_multi_step(st)
    else:
        launches_per_step = ncalls * r.launches_per_call
        step_fn = r.step

    stream = torch.cuda.Stream(device)
    warm(step_fn, args.warmup, stream, torch)

    # Capture the timed steps as graphs of back-to-back launches.
    K = args.steps
    graphs = []
    remaining = K
    while remaining > 0:
        s = min(graph_chunk(r.period), remaining)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            cs = torch.cuda.current_stream().cuda_stream
            for _ in range(s):
                step_fn(cs)
        graphs.append(g)
        remaining -= s
    # one untimed replay of every graph (first-launch costs)
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()

    bus = None
    try:
        pr = torch.cuda.get_device_properties(device)
        bus = f"{int(pr.pci_bus_id):02x}:{int(pr.pci_device_id):02x}."
    except Exception:
        pass
    sampler = ClockSampler(bus)
    if world > 1:
        torch.distributed.barrier()
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for g in graphs:
            g.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    total_ms = t0.elapsed_time(t1)
    del graphs
    assert sg.device_error(device) == 0, "a kernel reported a device-side error"

    step_bytes, step_flops, step_rows = step_accounting(p)
    calls_per_step = 1 if fused_step else ncalls
    call_bytes = step_bytes if fused_step else call_accounting(p, 0)[0]
    total_ms, all_bytes, all_flops, all_tokens = reduce_over_ranks(total_ms, step_bytes, step_flops,
                                                                   p.total_tokens, device, world)
    ms_per_step = total_ms / K
    value = all_bytes * K / (total_ms * 1e-3) / 1e9
    avg_launch_ms = total_ms / (K * calls_per_step)
    achieved = call_bytes / (avg_launch_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peak()

    # ---- the same step with an L2 flush before every step, median of FLUSH_STEPS
    flushed = None
    if not args.no_flush:
        fl = time_flushed(step_fn, FLUSH_STEPS, stream, torch, device)
        med = statistics.median(fl)
        med = reduce_over_ranks(med, 0, 0, 0, device, world)[0]
        assert sg.device_error(device) == 0, "a kernel reported a device-side error"
        f_ach = call_bytes / (med / calls_per_step * 1e-3) / 1e9
        flushed = {"ms_per_step_median": med, "ms_per_step_min": min(fl), "ms_per_step_max": max(fl),
                   "steps": FLUSH_STEPS, "value": all_bytes / (med * 1e-3) / 1e9, "unit": "GB/s",
                   "achieved": f_ach, "frac": f_ach / peak,
                   "note": f"a {FLUSH_BYTES >> 20} MiB write before every step; CUDA events around each step "
                           f"alone (eager launches, no graph); median over steps"}

    # ---- eager back-to-back steps (no graph) and the host time inside the calls
    eager = None
    if not args.no_eager:
        warm(step_fn, 3, stream, torch)
        dev_ms, host_ms = time_eager(step_fn, EAGER_STEPS, stream, torch)
        dev_ms = reduce_over_ranks(dev_ms, 0, 0, 0, device, world)[0]
        assert sg.device_error(device) == 0, "a kernel reported a device-side error"
        e_ach = call_bytes / (dev_ms / (EAGER_STEPS * calls_per_step) * 1e-3) / 1e9
        eager = {"ms_per_step": dev_ms / EAGER_STEPS, "steps": EAGER_STEPS,
                 "value": all_bytes * EAGER_STEPS / (dev_ms * 1e-3) / 1e9, "unit": "GB/s",
                 "achieved": e_ach, "frac": e_ach / peak,
                 "host_us_per_call": host_ms * 1e3 / (EAGER_STEPS * calls_per_step),
                 "note": "back-to-back calls through the C ABI without a CUDA graph; host_us_per_call is the "
                         "host time from entry to return of one call (validation, plan, tensor maps, launch)"}

    # ---- end to end: pinned host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        phx, phy = r.hx.pin_memory(), r.hy.pin_memory()
        phws = [w.pin_memory() for w in r.hws]
        phmeta = [m.pin_memory() for m in r.hmeta]
        out_host = torch.empty_like(phy).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in [phx, phy, *phws, *phmeta])
        d2h = out_host.numel() * out_host.element_size()
        E = args.e2e_steps
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(E):
                r.x.copy_(phx, non_blocking=True)
                r.y.copy_(phy, non_blocking=True)
                for w, pw in zip(r.ws, phws):
                    w.copy_(pw, non_blocking=True)
                for m, pm in zip(r.meta, phmeta):
                    m.copy_(pm, non_blocking=True)
                if fused_step:
                    step_fn(stream.cuda_stream)
                else:
                    r.step_first_copy(stream.cuda_stream)
                out_host.copy_(r.y, non_blocking=True)
            e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        e2e_ms = reduce_over_ranks(e2e_ms, 0, 0, 0, device, world)[0]
        e2e = {"value": all_bytes * E / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms / E, "steps": E}

    # ---- the same step as ONE fused multi-slice launch (several slices only)
    fused = None
    if ncalls > 1 and not args.no_fused and not fused_step:
        run_multi = r.multi_call()
        fv, fl = sg.plan_multi_slice(r.x, r.ws, r.y, *r.meta, p.batches, p.max_seq_len,
                                     [c.slice_offset for c in p.calls], p.add_inputs)
        warm(run_multi, args.warmup, stream, torch)
        if world > 1:
            torch.distributed.barrier()
        fms = time_graph_region(run_multi, K, stream, torch)
        fms = reduce_over_ranks(fms, 0, 0, 0, device, world)[0]
        assert sg.device_error(device) == 0, "a kernel reported a device-side error"
        f_ach = step_bytes / (fms / K * 1e-3) / 1e9
        fused = {"entry_point": "sgmv_expand_multi_slice", "launches_per_step": fl,
                 "variant": {1: "simt", 2: "tc"}.get(fv, "per-slice"),
                 "ms_per_step": fms / K, "value": all_bytes * K / (fms * 1e-3) / 1e9, "unit": "GB/s",
                 "achieved": f_ach, "frac": f_ach / peak, "bytes_per_launch": step_bytes / max(fl, 1),
                 "note": "all slices of a step in one call; same bytes as the separate calls"}

    # ---- the other workloads, each graph-timed on its own inputs (rank 0's figures)
    configs = None
    if not args.no_configs:
        configs = {}
        main_call_us = avg_launch_ms * 1e3
        configs[args.workload] = {
            "workload": WORKLOAD_TEXT[args.workload], "variant": r.variant, "calls_per_step": calls_per_step,
            "us_per_call": main_call_us, "gb_s": achieved, "frac": achieved / peak,
            "tokens_per_s": p.total_tokens * K / (total_ms * 1e-3), "tflops": step_flops * K / (total_ms * 1e-3) / 1e12,
            "bytes_per_call": call_bytes, "steps": K, "traffic": recorded_traffic(args.workload, r.kernel_family),
            "note": "the headline figures above"}
        for name in CONFIG_WORKLOADS:
            if name == args.workload:
                continue
            configs[name] = secondary_entry(name, args.seed + rank, max(SECONDARY_STEPS, K), args.warmup, device,
                                            peak)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(p, budget_s=args.cpu_seconds)

    trafrec = recorded_traffic_split(args.workload, r.kernel_family)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": p.w_dt, "accumulate": "f32",
        "data": "synthetic (seeded numpy; inputs resident in HBM)",
        "config": workload_config(p, args.workload, world, fused_step),
        "variant": r.variant,
        "timing": f"CUDA graphs of <= {STEPS_PER_GRAPH} steps; events around the timed region",
        "tokens_per_s": all_tokens * K / (total_ms * 1e-3),
        "tokens_per_s_note": "batch tokens per second, all ranks (a step updates every slice of every token)",
        "tflops": all_flops * K / (total_ms * 1e-3) / 1e12,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": trafrec["traffic"] if trafrec else None,
                     "dram_read": trafrec["read"] if trafrec else None,
                     "dram_write": trafrec["write"] if trafrec else None,
                     "traffic_note": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch of the current "
                                     "kernel source; reads are complete, writes still dirty in L2 when the launch "
                                     "ends are not counted, so dram_read is the figure to hold against the "
                                     "algorithmic reads",
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_kind == "measured" else "fallback 6650 GB/s",
                     "kernel": f"{ {'bgmv': 'bgmv_expand_slice', 'shrink': 'sgmv_shrink'}.get(p.op, 'sgmv_expand_slice') } "
                               f"({r.variant}{', %d H splits + reduction' % r.shrink_splits if r.shrink_splits > 1 else ''})",
                     "launch_ms_avg": avg_launch_ms, "bytes_per_launch": call_bytes,
                     "launch_sm_cycles": (avg_launch_ms * 1e-3 * clocks["sm_mhz"] * 1e6
                                          if clocks and clocks.get("sm_mhz") else None),
                     "launches_timed": K * calls_per_step,
                     "launch_ms_note": "timed region / calls (back-to-back calls, gaps included; launch_sm_cycles = "
                                       "that time x the median SM clock sampled during the region; a split shrink "
                                       "call is its main kernel plus the reduction)"},
        "gpu_launches": K * launches_per_step,
        "clocks": clocks,
        "l2_flushed": flushed,
        "eager": eager,
        "fused_multi_slice": fused,
        "configs": configs,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "when": datetime.datetime.now(datetime.timezone.utc).isoformat(),
    }
    return line


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(p, rows_budget, rng):
    """A compact problem made of the first rows of randomly chosen sequences of
    the workload (about rows_budget active rows): the chosen rows of x and of
    the output are copied out, and the segments renumbered onto them."""
    A = p.calls[0].w.shape[0]
    valid = [b for b in range(p.batches) if 0 <= p.lora_idx[b] < A and p.seq_len[b] > 0]
    order = rng.permutation(valid)
    rows, lens, idx = [], [], []
    left = rows_budget
    for b in order:
        if left <= 0:
            break
        take = int(min(p.seq_len[b], left))
        rows.append(np.arange(p.seq_start[b], p.seq_start[b] + take))
        lens.append(take)
        idx.append(p.lora_idx[b])
        left -= take
    rows = np.concatenate(rows)
    lens = np.array(lens, np.int64)
    return gen.Problem(p.name, np.ascontiguousarray(p.x[rows]), p.x_dt, p.w_dt,
                       np.ascontiguousarray(p.y0[rows]), p.out_dt, gen.exclusive_cumsum(lens), lens,
                       np.array(idx, np.int64), p.add_inputs, p.calls)


def run_oracle_sample(sub, nthreads):
    import oracle
    out = sub.y0
    t0 = time.perf_counter()
    for c in range(len(sub.calls)):
        out = oracle.run_problem(sub, out=out, call=c, nthreads=nthreads)
    return time.perf_counter() - t0, sub


def cpu_baseline(p, budget_s=15.0, nthreads=None):
    import oracle
    nthreads = nthreads or oracle.max_threads()
    rng = np.random.default_rng(0)
    # calibrate on a small sample, then size the measured one to the budget
    dt, sub = run_oracle_sample(oracle_sample(p, 8, rng), nthreads)
    rows_per_s = max(int(sub.seq_len.sum()), 1) / max(dt, 1e-6)
    rows = int(max(8, min(rows_per_s * budget_s, p.seq_len.sum())))
    dt, sub = run_oracle_sample(oracle_sample(p, rows, np.random.default_rng(1)), nthreads)
    b, _, r = step_accounting(sub)
    return {"value": b / dt / 1e9, "unit": "GB/s", "cores": int(nthreads), "kind": "oracle",
            "seconds": dt,
            "sample": f"{int(sub.seq_len.sum())} active rows from {len(sub.seq_len)} sequences of the same "
                      f"workload, all {len(p.calls)} slices (fp64 C triple loop, OpenMP over rows)"}


def bench_reference(args, rank, world):
    """The CPU oracle, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    p = gen.WORKLOADS[args.workload](seed=args.seed)
    nthreads = oracle.max_threads()
    # rows per step so that warm-up + steps take about args.cpu_seconds
    dt, sub = run_oracle_sample(oracle_sample(p, 8, np.random.default_rng(0)), nthreads)
    rows_per_s = max(int(sub.seq_len.sum()), 1) / max(dt, 1e-6)
    per_step = int(max(1, min(rows_per_s * args.cpu_seconds / max(args.steps + args.warmup, 1),
                              p.seq_len.sum())))
    rng = np.random.default_rng(2)
    for _ in range(args.warmup):
        run_oracle_sample(oracle_sample(p, per_step, rng), nthreads)
    tot_t = 0.0
    tot_b = 0
    rows = 0
    for _ in range(args.steps):
        dt, sub = run_oracle_sample(oracle_sample(p, per_step, rng), nthreads)
        b, _, r = step_accounting(sub)
        tot_t += dt
        tot_b += b
        rows += int(sub.seq_len.sum())
    value = tot_b / tot_t / 1e9
    sample_txt = (f"{per_step} active rows per step drawn from the {args.workload} workload, all "
                  f"{len(p.calls)} slices; fp64 C triple loop with OpenMP over rows")
    return {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_t / max(args.steps, 1) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": workload_config(p, args.workload, world),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": nthreads, "kind": "oracle",
                             "sample": sample_txt},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(gen.WORKLOADS), default="qkv_prefill")
    ap.add_argument("--variant", choices=["auto", "simt", "tc"], default="auto")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fused", action="store_true",
                    help="skip the extra timing of the step as one multi-slice call")
    ap.add_argument("--step", choices=["calls", "fused"], default="calls",
                    help="time each step as separate slice calls (default) or as one multi-slice call")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-configs", action="store_true", help="skip the figures of the other workloads")
    ap.add_argument("--no-flush", action="store_true", help="skip the L2-flushed median timing")
    ap.add_argument("--no-eager", action="store_true", help="skip the eager (no graph) timing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = bench_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    device = torch.device("cuda", local)
    if world > 1:
        torch.cuda.set_device(device)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        line = bench_ours(args, rank, world, device)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
