#!/usr/bin/env python
"""Benchmark of the residual-compression codec on B200 (one JSON line).

A step is one denoising step of the codec over every slot of the workload:
cf_compress (residual + error feedback + k-bit group quantisation + packing,
one grouped launch) followed by cf_decompress (unpack + dequantise +
accumulate, one grouped launch), on synthetic activations shaped like the
FLUX.1-dev patch-parallel shard (57 blocks x 1152 tokens x 3072 channels,
bf16, 2-bit codes, groups of 128).  The warmup step 0 runs before timing.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cf|reference]

Under torchrun (N > 1) every rank runs the whole workload on its own GPU
(the codec has no cross-slot exchange: weak scaling, no data-path
collective); rank 0 prints the line with the max time over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "codec GB/s of activation input and % of B200 HBM roofline (1 GPU)"
FALLBACK_HBM_GBS = 6650.0


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def alg_bytes_per_elem(bits, group):
    """Algorithmic HBM bytes per activation element (compress, decompress).

    compress  : read X (2), base (2), E (4); write base (2), E (4), codes k/8,
                scales 4/G
    decompress: read codes k/8, scales 4/G, C (4); write C (4)
    """
    payload = bits / 8 + 4 / group
    return 2 + 2 + 4 + 2 + 4 + payload, payload + 4 + 4


def bf16_peak():
    """Dense bf16 tensor peak (TFLOP/s): the measured burst figure, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def source_hash(src="cf_quant.cu"):
    p = os.path.join(ROOT, "activation_residual_compression_02_b200", "csrc", src)
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel, src="cf_quant.cu", field="dram_bytes_per_launch"):
    """A recorded ncu figure of a kernel (by default its DRAM bytes per launch,
    per call for the whole low-rank call) from profiles/traffic.json, reported
    only while that capture's source file is the one built here."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(kernel)
        if e and e.get("source_sha") == source_hash(src) and e.get(field) is not None:
            return float(e[field])
    except Exception:
        pass
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while ``active``.

    The NVML handle is found by the GPU's UUID (else its PCI bus id), since
    NVML numbers devices physically and ignores CUDA_VISIBLE_DEVICES.  Samples
    are kept only while ``active`` is set, i.e. inside the timed regions.
    """

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, dev_index):
        self.samples = []
        self.ok = False
        self.reasons = set()
        self.active = False
        self.how = None
        self._stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h, self.how = self._handle(pynvml, dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    @staticmethod
    def _handle(nv, dev_index):
        props = torch.cuda.get_device_properties(dev_index)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            want = str(uuid).lower().replace("gpu-", "")
            for i in range(nv.nvmlDeviceGetCount()):
                h = nv.nvmlDeviceGetHandleByIndex(i)
                u = nv.nvmlDeviceGetUUID(h)
                u = (u.decode() if isinstance(u, bytes) else u).lower().replace("gpu-", "")
                if u == want:
                    return h, "uuid"
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            busid = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), bus, getattr(props, "pci_device_id", 0))
            return nv.nvmlDeviceGetHandleByPciBusId_v2(busid), "pci_bus_id"
        raise RuntimeError("cannot match the CUDA device to an NVML device")

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            if self.active:
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    if self.active:
                        self.samples.append(mhz)
                        for bit, name in self.REASONS.items():
                            if r & bit:
                                self.reasons.add(name)
                except Exception:
                    pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def __enter__(self):
        self.start()
        self.active = True
        return self

    def __exit__(self, *a):
        self.active = False
        self.stop()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples), "nvml_device": self.how,
                "window": "every timed region of this run"}


class Timed:
    """Marks a timed region for the clock sampler (samples are kept only inside)."""

    def __init__(self, clk):
        self.clk = clk

    def __enter__(self):
        if self.clk is not None:
            self.clk.active = True
        return self

    def __exit__(self, *a):
        if self.clk is not None:
            self.clk.active = False


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# --------------------------------------------------------------- CPU oracle

def oracle_run(w, xs_host, threads):
    """Time the oracle (compress + decompress) over host inputs
    ``xs_host[slot] = [X_0, X_1, ...]`` (raw bf16 bits); step 0 (the warmup)
    is untimed.  Returns (seconds, elements of the timed steps)."""
    import concurrent.futures

    import oracle

    oracle.build()
    slots = sorted(xs_host)
    states = {s: oracle.QuantSlot(w.bits, w.group) for s in slots}
    for s in slots:
        states[s].step(0, xs_host[s][0])

    def work(s):
        for t in range(1, len(xs_host[s])):
            states[s].step(t, xs_host[s][t])

    t0 = time.perf_counter()
    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(work, slots))
    dt = time.perf_counter() - t0
    elems = sum(x.size for s in slots for x in xs_host[s][1:])
    return dt, elems


def host_inputs(w, rows, steps, seed=0):
    """Inputs of `steps` steps (warmup included) for `rows` token rows of every slot, generated on the host."""
    import numpy as np

    sub = w.scaled(rows=rows)
    return {s: [synth.bf16_bits(x).numpy().view(np.uint16).ravel().copy()
                for x in synth.activations(sub, s, steps, seed=seed)] for s in range(w.slots)}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    import platform

    return platform.processor() or "unknown"


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------- main

def run_reference(args, w):
    # the oracle runs on rank 0's host cores only; other ranks exit without work
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    cores = cpu_cores()
    steps = args.steps + args.warmup
    budget = args.budget
    # about 15 ns of oracle work per element per step on one core; size the
    # per-step row sample so that the whole run stays within the budget
    per_step_elems = budget / steps * cores / 15e-9
    rows = int(max(1, min(w.rows, per_step_elems // (w.slots * w.cols))))
    xs = host_inputs(w, rows, 1 + args.warmup + args.steps, seed=1)
    warm = {s: v[:1 + args.warmup] for s, v in xs.items()}
    oracle_run(w, warm, cores)
    timed = {s: [v[0]] + v[1 + args.warmup:] for s, v in xs.items()}
    dt, elems = oracle_run(w, timed, cores)
    gbs = elems * 2 / dt / 1e9
    sample = f"{rows} token rows of each of the {w.slots} slots, {args.steps} compressed steps"
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def payload_summary(ctx, w):
    """What one compressed step sends per rank: the packed codes and scales of
    every slot (cf_payload_bytes) against the raw bf16 activations, i.e. the
    communication reduction the pages report (8-16x) for this workload's k and G."""
    pay = sum(ctx.payload_bytes(s) for s in range(w.slots))
    raw = w.elems * 2
    return {"bytes_per_step": pay, "raw_bf16_bytes_per_step": raw, "reduction": raw / pay,
            "bytes_per_elem": pay / w.elems}


def workload_config(w):
    return {
        "workload": f"{w.name}: {w.slots} slots x {w.rows} tokens x {w.cols} channels bf16, k={w.bits}, "
                    f"G={w.group}, error feedback, {w.steps} denoising steps",
        "slots": w.slots, "rows": w.rows, "cols": w.cols, "bits": w.bits, "group": w.group,
        "l2": "inputs larger than L2 (every step streams the whole state)",
    }


def run_cf(args, w):
    world, rank, local = dist_init()
    import activation_residual_compression_02_b200 as cf

    dev = torch.device("cuda", torch.cuda.current_device())
    clk = ClockSampler(torch.cuda.current_device()).start()
    shapes = [(w.rows, w.cols)] * w.slots
    ctx = cf.Context(shapes, bits=w.bits, group=w.group)
    st = cf.QuantState(shapes, w.bits, w.group, device=dev)
    n_elem = w.elems
    x_bytes = n_elem * 2

    # all inputs of the run resident in HBM before timing
    nsteps = min(w.steps, 1 + args.warmup + args.steps)
    streams = [synth.SlotStream(w, s, seed=rank, device=dev) for s in range(w.slots)]
    X = [[None] * w.slots for _ in range(nsteps)]
    for s in range(w.slots):
        for t in range(nsteps):
            X[t][s] = streams[s].next().reshape(-1)
        streams[s].state = None
    del streams
    torch.cuda.synchronize()

    def x_at(i):  # step index i >= 1 cycles through the compressed steps
        return X[1 + (i - 1) % (nsteps - 1)] if nsteps > 1 else X[0]

    stream = torch.cuda.current_stream()
    slots0 = st.slots(X[0])
    ctx.compress(slots0, 0)
    ctx.decompress(slots0, 0)
    slot_lists = [st.slots(x_at(i)) for i in range(1, min(nsteps, 1 + args.warmup + args.steps))]
    c_slots = [ctx._slots(sl) for sl in slot_lists]  # C slot arrays built once, outside the timing
    L = cf.lib()
    h = ctx.handle
    sh = stream.cuda_stream

    def step(i):
        arr = c_slots[(i - 1) % len(c_slots)]
        if L.cf_compress(h, arr, i, sh) != 0 or L.cf_decompress(h, arr, i, sh) != 0:
            raise RuntimeError(L.cf_last_error(h).decode())

    for i in range(1, args.warmup + 1):
        step(i)
    torch.cuda.synchronize()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with Timed(clk):
        start.record(stream)
        for k in range(args.steps):
            i = args.warmup + 1 + k
            arr = c_slots[(i - 1) % len(c_slots)]
            ev[k][0].record(stream)
            if L.cf_compress(h, arr, i, sh) != 0:
                raise RuntimeError(L.cf_last_error(h).decode())
            ev[k][1].record(stream)
            if L.cf_decompress(h, arr, i, sh) != 0:
                raise RuntimeError(L.cf_last_error(h).decode())
            ev[k][2].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    status = ctx.check()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    ms_local = start.elapsed_time(end)
    ms = max_over_ranks(ms_local, world)

    # ---- the same steps through cf_loopback (sender and receiver fused) ---
    lb = None
    if not args.no_loopback:
        for i in range(1, args.warmup + 1):
            if L.cf_loopback(h, c_slots[(i - 1) % len(c_slots)], i, sh) != 0:
                raise RuntimeError(L.cf_last_error(h).decode())
        barrier(world)
        torch.cuda.synchronize()
        l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with Timed(clk):
            l0.record(stream)
            for k in range(args.steps):
                i = args.warmup + 1 + k
                if L.cf_loopback(h, c_slots[(i - 1) % len(c_slots)], i, sh) != 0:
                    raise RuntimeError(L.cf_last_error(h).decode())
            l1.record(stream)
            torch.cuda.synchronize()
        lb_ms = max_over_ranks(l0.elapsed_time(l1), world) / args.steps
        lb_bytes = (22.0 + w.bits / 8 + 4 / w.group) * n_elem
        lb = {"ms_per_step": lb_ms, "value": world * x_bytes / (lb_ms * 1e-3) / 1e9, "unit": "GB/s",
              "alg_bytes_per_step": lb_bytes, "achieved": lb_bytes / (lb_ms * 1e-3) / 1e9,
              "frac": lb_bytes / (lb_ms * 1e-3) / 1e9 / hbm_peak()[0],
              "note": "cf_loopback: compress and decompress of a step in one launch (both sides on this GPU)"}
    comp_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    deco_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps

    # ---- receiver with the bf16 reconstruction (recon), same payload ------
    # The decompress of the last timed step again, K times, with every slot's
    # recon set; beside it the same decompress followed by torch's fp32 -> bf16
    # cast of the caches (the separate pass recon replaces).
    rc = None
    if not args.no_recon:
        last = (args.warmup + args.steps - 1) % len(c_slots)
        recon_all = torch.empty(st.cache_all.numel(), dtype=torch.bfloat16, device=dev)
        r_list = st.slots(x_at(last + 1))
        for sl_, c_ in zip(r_list, st.cache):
            # recon of a slot at its cache's element offset (16-byte aligned: cols % 8 == 0)
            o = c_.storage_offset() - st.cache_all.storage_offset()
            sl_.recon = recon_all[o:o + c_.numel()]
        r_arr = ctx._slots(r_list)
        i_dec = args.warmup + args.steps

        def deco(arr):
            if L.cf_decompress(h, arr, i_dec, sh) != 0:
                raise RuntimeError(L.cf_last_error(h).decode())

        for _ in range(args.warmup):
            deco(r_arr)
        barrier(world)
        torch.cuda.synchronize()
        r0, r1, r2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        with Timed(clk):
            r0.record(stream)
            for _ in range(args.steps):
                deco(r_arr)
            r1.record(stream)
            for _ in range(args.steps):
                deco(c_slots[last])
                recon_all.copy_(st.cache_all)
            r2.record(stream)
            torch.cuda.synchronize()
        if ctx.check() != 0:
            raise RuntimeError("device status in the recon run")
        r_ms = max_over_ranks(r0.elapsed_time(r1), world) / args.steps
        cast_ms = max_over_ranks(r1.elapsed_time(r2), world) / args.steps
        _, bd_ = alg_bytes_per_elem(w.bits, w.group)
        r_bytes = (bd_ + 2) * n_elem
        rc = {"ms_per_launch": r_ms, "alg_bytes_per_launch": r_bytes, "achieved": r_bytes / (r_ms * 1e-3) / 1e9,
              "frac": r_bytes / (r_ms * 1e-3) / 1e9 / hbm_peak()[0], "decompress_then_cast_ms": cast_ms,
              "note": "cf_decompress with recon: C += deq and recon = bf16(C) in one pass (bd + 2 B/elt); "
                      "decompress_then_cast_ms: the same decompress followed by torch's cast of C to bf16"}
        del recon_all, r_arr, r_list
    ms_per_step = ms / args.steps
    value = world * x_bytes / (ms_per_step * 1e-3) / 1e9

    # ---- the warmup step (step 0 again: base, E and C from X_0) -----------
    # Once per generation in a deployment; timed here so that the whole run
    # (1 warmup + 27 compressed steps for FLUX) can be costed.
    a0 = ctx._slots(slots0)
    for _ in range(2):
        if L.cf_compress(h, a0, 0, sh) != 0 or L.cf_decompress(h, a0, 0, sh) != 0:
            raise RuntimeError(L.cf_last_error(h).decode())
    barrier(world)
    torch.cuda.synchronize()
    wev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    with Timed(clk):
        for k in range(args.steps):
            wev[k][0].record(stream)
            L.cf_compress(h, a0, 0, sh)
            wev[k][1].record(stream)
            L.cf_decompress(h, a0, 0, sh)
            wev[k][2].record(stream)
        torch.cuda.synchronize()
    ws_ms = sum(e[0].elapsed_time(e[1]) for e in wev) / args.steps
    wr_ms = sum(e[1].elapsed_time(e[2]) for e in wev) / args.steps
    warm = {"sender_ms": ws_ms, "receiver_ms": wr_ms,
            "sender_frac": 8 * n_elem / (ws_ms * 1e-3) / 1e9 / hbm_peak()[0],
            "receiver_frac": 6 * n_elem / (wr_ms * 1e-3) / 1e9 / hbm_peak()[0],
            "note": "step 0: base = X, E = 0 (8 B/elt); C = float(X) (6 B/elt)"}

    bc, bd = alg_bytes_per_elem(w.bits, w.group)
    peak, peak_kind = hbm_peak()
    ach_c = bc * n_elem / (comp_ms * 1e-3) / 1e9
    ach_d = bd * n_elem / (deco_ms * 1e-3) / 1e9
    ach_pair = (bc + bd) * n_elem / (ms_per_step * 1e-3) / 1e9

    # ---- the lean state (E and C in bf16), same inputs -------------------
    lean = None
    if not args.no_lean:
        lctx = cf.Context(shapes, bits=w.bits, group=w.group, state_bf16=1)
        lst = cf.QuantState(shapes, w.bits, w.group, device=dev, lean=True)
        l_arrays = [lctx._slots(lst.slots(x_at(i))) for i in range(1, min(nsteps, 1 + args.warmup + args.steps))]
        l0_arr = lctx._slots(lst.slots(X[0]))
        lh = lctx.handle

        def lean_step(i, arr):
            if L.cf_compress(lh, arr, i, sh) != 0 or L.cf_decompress(lh, arr, i, sh) != 0:
                raise RuntimeError(L.cf_last_error(lh).decode())

        lean_step(0, l0_arr)
        for i in range(1, args.warmup + 1):
            lean_step(i, l_arrays[(i - 1) % len(l_arrays)])
        barrier(world)
        torch.cuda.synchronize()
        q0e, q1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        lev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        with Timed(clk):
            q0e.record(stream)
            for k in range(args.steps):
                i = args.warmup + 1 + k
                arr = l_arrays[(i - 1) % len(l_arrays)]
                lev[k][0].record(stream)
                if L.cf_compress(lh, arr, i, sh) != 0:
                    raise RuntimeError(L.cf_last_error(lh).decode())
                lev[k][1].record(stream)
                if L.cf_decompress(lh, arr, i, sh) != 0:
                    raise RuntimeError(L.cf_last_error(lh).decode())
                lev[k][2].record(stream)
            q1e.record(stream)
            torch.cuda.synchronize()
        if lctx.check() != 0:
            raise RuntimeError("device status in the lean run")
        lean_ms = max_over_ranks(q0e.elapsed_time(q1e), world) / args.steps
        lc_ms = sum(e[0].elapsed_time(e[1]) for e in lev) / args.steps
        ld_ms = sum(e[1].elapsed_time(e[2]) for e in lev) / args.steps
        pay = w.bits / 8 + 4 / w.group
        lc_b, ld_b = (2 + 2 + 2 + 2 + 2 + pay) * n_elem, (pay + 2 + 2) * n_elem
        lean_bytes = lc_b + ld_b
        lean = {"ms_per_step": lean_ms, "value": world * x_bytes / (lean_ms * 1e-3) / 1e9, "unit": "GB/s",
                "alg_bytes_per_step": lean_bytes, "achieved": lean_bytes / (lean_ms * 1e-3) / 1e9,
                "frac": lean_bytes / (lean_ms * 1e-3) / 1e9 / peak,
                "compress": {"ms_per_launch": lc_ms, "frac": lc_b / (lc_ms * 1e-3) / 1e9 / peak},
                "decompress": {"ms_per_launch": ld_ms, "frac": ld_b / (ld_ms * 1e-3) / 1e9 / peak},
                "note": "state_bf16=1: E and C kept in bf16 (14.56 B/elt for compress + decompress)"}
        del lctx, lst, l_arrays

    # ---- end to end through the public API, host buffers -----------------
    # Pinned host activations in, payload (codes + scales) back to pinned host
    # memory, every step; HostStreamCodec overlaps the host-to-device copy of
    # step t+1 and the device-to-host copy of step t-1 with the codec on step t.
    e2e = None
    if not args.no_e2e:
        hc = cf.HostStreamCodec(shapes, bits=w.bits, group=w.group, device=dev)
        n_host = min(4, nsteps)
        host_x = []
        for j in range(n_host):
            buf, views = hc.st.activation_buffer(pin=True)
            for s_, v in enumerate(views):
                v.copy_(X[j][s_])
            host_x.append(buf)
        host_pay = [hc.st.payload_buffers(pin=True) for _ in range(2)]
        h2d = x_bytes
        d2h = host_pay[0][0].numel() + 4 * host_pay[0][2].numel()
        e2e_steps = max(3, min(args.steps, 30))

        def e2e_step(t):
            hp = host_pay[t % 2]
            hc.step(t, host_x[t % n_host], hp[0], hp[2])

        e2e_step(0)
        for t in range(1, 3):
            e2e_step(t)
        hc.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with Timed(clk):
            e0.record(hc.s_h2d)
            for t in range(3, 3 + e2e_steps):
                e2e_step(t)
            for s_ in (hc.s_codec, hc.s_d2h):
                ev = torch.cuda.Event()
                ev.record(s_)
                hc.s_h2d.wait_event(ev)
            e1.record(hc.s_h2d)
            hc.synchronize()
        if hc.check() != 0:
            raise RuntimeError("device status after the e2e run")
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
        e2e = {"value": world * x_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
               "host_inputs": f"{n_host} pinned host copies of the step inputs, cycled; copies overlapped with "
                              "the codec on three streams"}
        del hc
    status = ctx.check()
    if status != 0:
        raise RuntimeError(f"device status {status}")

    # ---- CPU oracle on a bounded sample (rank 0, N = 1) -------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        import numpy as np

        cores = cpu_cores()
        csteps = min(args.cpu_steps, nsteps - 1)
        xs_host = {s: [X[t][s].view(torch.int16).cpu().numpy().view(np.uint16).copy() for t in range(1 + csteps)]
                   for s in range(w.slots)}
        dt, elems = oracle_run(w, xs_host, cores)
        cpu = {"value": elems * 2 / dt / 1e9, "unit": "GB/s", "cores": cores, "cpu_model": cpu_model(),
               "kind": "oracle",
               "sample": f"the whole workload ({w.slots} slots x {w.rows} x {w.cols}) for {csteps} compressed "
                         f"steps after the warmup (compress + decompress, {elems} elements), one slot per host "
                         f"thread, {cores} threads, {dt:.1f} s wall"}

    # ---- the other workloads of the codec, as extra keys of this line ----
    # The CogVideoX-shaped and stress steps (quantised), the low-rank call
    # (Algorithm 3 + apply on 57 x 4608 x 3072 fp32), and the attention that
    # consumes a received CogVideoX-shaped K/V shard, each timed the same way.
    cog = stress = lowrank = attention = None
    if not args.no_extra:
        del X, slot_lists, c_slots, slots0, st
        torch.cuda.empty_cache()
        cog = quant_extra(args, synth.COGVIDEOX, world, rank, clk, min(args.steps, 30))
        stress = quant_extra(args, synth.STRESS, world, rank, clk, min(args.steps, 10))
        lowrank = lowrank_measure(args, synth.LOWRANK, world, rank, clk, min(args.steps, 20),
                                  0 if args.no_cpu else 4)
        if lowrank.get("cpu_baseline"):
            lowrank["cpu_baseline"]["sample"] += " (a bounded sample: the run stays short)"
        torch.cuda.empty_cache()
        attention = attention_measure(args, synth.COGVIDEOX, world, rank, clk, min(args.steps, 10))
    clk.stop()

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": workload_config(w),
        "roofline": {"bound": "hbm", "kernel": "compress (residual+EF+quantise+pack, grouped)",
                     "achieved": ach_c, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": ach_c / peak, "traffic": recorded_traffic("compress"),
                     "alg_bytes_per_launch": bc * n_elem, "ms_per_launch": comp_ms},
        "roofline_decompress": {"bound": "hbm", "achieved": ach_d, "peak": peak, "unit": "GB/s",
                                "frac": ach_d / peak, "traffic": recorded_traffic("decompress"),
                                "alg_bytes_per_launch": bd * n_elem, "ms_per_launch": deco_ms},
        "roofline_step": {"achieved": ach_pair, "frac": ach_pair / peak, "frac_of_8tbs": ach_pair / 8000.0,
                          "alg_bytes_per_step": (bc + bd) * n_elem},
        "loopback": lb, "lean_state": lean, "recon": rc, "warmup_step": warm,
        "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": 2 * args.steps,
        "payload": payload_summary(ctx, w),
        "cogvideox": cog, "stress": stress, "lowrank": lowrank, "attention": attention,
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def lowrank_measure(args, w, world, rank, clk, steps, cpu_mats, through_slots=False, warm_start=False, precision=0):
    """Algorithm 3 on the low-rank workload (k fp32 residual matrices of
    m x n, rank r, T iterations, Gaussian start blocks) through cf_lowrank,
    with the error buffer E = A - U R V^T written: a step of the low-rank
    codec's sender on given residuals.  Times `steps` calls with CUDA events,
    then the same calls again with per-launch tracing (cf_trace).  Returns the
    fields of a bench line (without the line's own keys)."""
    import activation_residual_compression_02_b200 as cf

    dev = torch.device("cuda", torch.cuda.current_device())
    m, n, r, T, k = w.rows, w.cols, w.rank, w.iters, w.slots
    if warm_start:
        T = 1      # each call starts from the previous call's V
    ctx = cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=r, iters=T, precision=precision)
    ws = torch.empty(ctx.lowrank_workspace_bytes(k, m, n), dtype=torch.uint8, device=dev)
    ctx.set_workspace(ws)
    A = [synth.lowrank_matrix(m, n, r, mat=i, seed=rank, device=dev) for i in range(k)]
    Q0 = [synth.q0(n, r, seed=rank, mat=i, device=dev) for i in range(k)]
    U = [torch.empty(m, r, device=dev) for _ in range(k)]
    R = [torch.empty(r, r, device=dev) for _ in range(k)]
    V = [torch.empty(n, r, device=dev) for _ in range(k)]
    E = [torch.empty(m, n, device=dev) for _ in range(k)]
    stream = torch.cuda.current_stream()
    ctx.lowrank(A, Q0, U, R, V, E)
    start_block = V if warm_start else Q0   # warm start: V doubles as the next start block
    for _ in range(args.warmup):
        ctx.lowrank(A, start_block, U, R, V, E)
    torch.cuda.synchronize()
    assert ctx.check() == 0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with Timed(clk):
        start.record(stream)
        for _ in range(steps):
            ctx.lowrank(A, start_block, U, R, V, E)
        end.record(stream)
        torch.cuda.synchronize()
    status = ctx.check()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    ms = max_over_ranks(start.elapsed_time(end), world) / steps

    # ---- the same calls again with per-launch tracing (cf_trace_*) -------
    # CUDA events around every kernel on the launching stream give each
    # kernel's live duration; the roofline line is the dominant kernel's.
    ctx.trace(True)
    with Timed(clk):
        for _ in range(steps):
            ctx.lowrank(A, start_block, U, R, V, E)
        torch.cuda.synchronize()
    trace = ctx.trace_read()
    ctx.trace(False)
    for e in trace:
        e["ms_per_launch"] = max_over_ranks(e["total_ms"] / e["launches"], world)
        e["launches_per_call"] = e["launches"] // steps
    dom = max(trace, key=lambda e: e["total_ms"] * 1.0)
    elems = k * m * n
    peak, peak_kind = hbm_peak()
    alg_bytes = elems * (4 + 4)          # A read once, E written once
    # one product with A: A read once, plus the r-column blocks (Q^T or P^T read, P^T or Z written; padded to rp)
    rp = 16 if r <= 16 else 32
    gemm_bytes = elems * 4 + k * (m + n) * rp * 4
    if not dom["kernel"].startswith("k_gemm"):   # the apply: A read, E written
        gemm_bytes = elems * 8
    sched_bytes = elems * (4 * (2 * T + 2) + 4)   # A read by each of the 2T+1 products and the apply, E written
    flops = 2.0 * (2 * T + 1) * m * n * r * k + 2.0 * m * n * r * k
    full_size = (k, m, n, r, w.iters) == (57, 4608, 3072, 16, 2) and not warm_start and precision == 0

    # ---- low-rank mode through cf_compress / cf_decompress ---------------
    # The same shapes as bf16 activation slots: each compressed step first
    # materialises A = (X - base) + E in fp32 (k_residual_f32), then runs the
    # call above on it; the receiver adds U R V^T to its cache.
    lr_mode = None
    if through_slots:
        shapes = [(m, n)] * k
        mctx = cf.Context(shapes, mode=cf.CF_MODE_LOWRANK, rank=r, iters=T, precision=precision)
        mws = torch.empty(mctx.workspace_bytes(), dtype=torch.uint8, device=dev)
        mctx.set_workspace(mws)
        wq = synth.FLUX.scaled(slots=k, rows=m, cols=n)
        sst = [synth.SlotStream(wq, i, seed=rank, device=dev) for i in range(k)]
        Xs = [[st_.next().reshape(-1) for st_ in sst] for _ in range(6)]
        del sst
        mb = [torch.empty(m * n, dtype=torch.bfloat16, device=dev) for _ in range(k)]
        me = [torch.empty(m * n, device=dev) for _ in range(k)]
        mc = [torch.empty(m * n, device=dev) for _ in range(k)]
        arrs = [mctx._slots([cf.Slot(x=Xs[j][i], base=mb[i], err=me[i], cache=mc[i], q0=Q0[i], U=U[i], R=R[i],
                                     V=V[i]) for i in range(k)]) for j in range(6)]
        L, h, sh = cf.lib(), mctx.handle, stream.cuda_stream

        def mstep(i, ev=None):
            arr = arrs[0] if i == 0 else arrs[1 + (i - 1) % 5]
            if ev:
                ev[0].record(stream)
            if L.cf_compress(h, arr, i, sh) != 0:
                raise RuntimeError(L.cf_last_error(h).decode())
            if ev:
                ev[1].record(stream)
            if L.cf_decompress(h, arr, i, sh) != 0:
                raise RuntimeError(L.cf_last_error(h).decode())
            if ev:
                ev[2].record(stream)

        for i in range(args.warmup + 1):
            mstep(i)
        torch.cuda.synchronize()
        barrier(world)
        mev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        with Timed(clk):
            for j in range(steps):
                mstep(args.warmup + 1 + j, mev[j])
            torch.cuda.synchronize()
        if mctx.check() != 0:
            raise RuntimeError("device status in the low-rank mode run")
        c_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in mev) / steps, world)
        d_ms = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in mev) / steps, world)
        lr_mode = {"compress_ms": c_ms, "decompress_ms": d_ms, "ms_per_step": c_ms + d_ms,
                   "value": world * elems * 2 / ((c_ms + d_ms) * 1e-3) / 1e9, "unit": "GB/s of bf16 activations",
                   "residual_ms_est": c_ms - ms,
                   "residual_frac_est": 14 * elems / ((c_ms - ms) * 1e-3) / 1e9 / peak if c_ms > ms else None,
                   "decompress_frac": 8 * elems / (d_ms * 1e-3) / 1e9 / peak,
                   "note": "cf_compress = residual (14 B/elt: x, base, E read, A and base written) + the cf_lowrank "
                           "call timed above; residual_ms_est = compress_ms - that call; decompress: C += U R V^T "
                           "(8 B/elt)"}
        del mctx, mws, Xs, mb, me, mc, arrs

    cpu = None
    if rank == 0 and world == 1 and cpu_mats > 0:
        import concurrent.futures

        import oracle

        oracle.build()
        nsample = min(cpu_mats, k)
        Ah = [A[i].cpu().numpy() for i in range(nsample)]
        Qh = [Q0[i].cpu().numpy() for i in range(nsample)]

        def work(i):
            Uo, Ro, Vo = oracle.subspace_iteration(Ah[i], Qh[i], T)
            oracle.lowrank_apply(Ah[i], Uo, Ro, Vo)

        threads = min(cpu_cores(), nsample)
        t0 = time.perf_counter()
        with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(work, range(nsample)))
        dt = time.perf_counter() - t0
        cpu = {"value": nsample * m * n * 4 / dt / 1e9, "unit": "GB/s", "cores": threads,
               "cpu_model": cpu_model(), "kind": "oracle",
               "sample": f"{nsample} of the {k} matrices (Algorithm 3 in fp64 plus the apply), one matrix per host "
                         f"thread, {threads} threads, {dt:.1f} s wall"}
    out = {
        "value": world * elems * 4 / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms, "steps": steps,
        "warmup": args.warmup,
        "config": {"workload": f"lowrank: {k} matrices x {m} x {n} fp32, rank-{r} signal + 0.01 noise, r={r}, "
                               f"T={T}, " + ("warm start from the previous V" if warm_start else "Gaussian Q0")
                               + ", E = A - U R V^T written"
                               + {0: "", 1: ", TF32 products", 2: ", split (3xTF32) products"}[precision],
                   "l2": "inputs larger than L2 (3.2 GB of A per step)"},
        "roofline": {"bound": "hbm", "kernel": dom["kernel"],
                     "achieved": gemm_bytes / (dom["ms_per_launch"] * 1e-3) / 1e9, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": gemm_bytes / (dom["ms_per_launch"] * 1e-3) / 1e9 / peak,
                     "traffic": recorded_traffic("lowrank_gemm", "cf_subspace.cu") if full_size else None,
                     "tensor_pipe": recorded_traffic("lowrank_gemm", "cf_subspace.cu", "tensor_pipe_active")
                     if full_size else None,
                     "alg_bytes_per_launch": gemm_bytes, "ms_per_launch": dom["ms_per_launch"],
                     "note": "the dominant kernel, timed live by per-launch CUDA events (cf_trace); one launch "
                             "is one product with A over all matrices: A read once, the r-column blocks read and "
                             "written (a read-only stream can exceed the copy peak); tensor_pipe: the fraction of "
                             "cycles the tensor pipe was active (ncu sm__pipe_tensor_cycles_active) in the recorded "
                             "capture of the same source"},
        "roofline_call": {"kernel": "whole cf_lowrank call", "achieved": alg_bytes / (ms * 1e-3) / 1e9,
                          "frac": alg_bytes / (ms * 1e-3) / 1e9 / peak,
                          "traffic": recorded_traffic("lowrank_call", "cf_subspace.cu") if full_size else None,
                          "alg_bytes_per_step": alg_bytes, "tflops": flops / (ms * 1e-3) / 1e12,
                          "schedule_bytes_per_step": sched_bytes,
                          "schedule_frac": sched_bytes / (ms * 1e-3) / 1e9 / peak,
                          "note": "alg bytes count A once and E once; the schedule reads A from HBM in each of "
                                  "the 2T+1 products and in the apply"},
        "kernels": [{"kernel": e["kernel"], "launches_per_call": e["launches_per_call"],
                     "ms_per_launch": e["ms_per_launch"]} for e in trace],
        "gpu_launches": steps * sum(e["launches_per_call"] for e in trace), "cpu_baseline": cpu,
        "lowrank_mode": lr_mode,
        # what a step sends per matrix: U (m x r), R (r x r) and V (n x r) in fp32, against the bf16 activation
        "payload": {"bytes_per_step": k * (m * r + r * r + n * r) * 4, "raw_bf16_bytes_per_step": k * m * n * 2,
                    "reduction": (m * n * 2) / ((m * r + r * r + n * r) * 4)},
    }
    ctx.close()
    del A, Q0, U, R, V, E, ws
    torch.cuda.empty_cache()
    return out


def run_lowrank_bench(args, w):
    """The low-rank workload as the bench line (--workload lowrank)."""
    world, rank, local = dist_init()
    clk = ClockSampler(torch.cuda.current_device()).start()
    out = lowrank_measure(args, w, world, rank, clk, args.steps, 0 if args.no_cpu else w.slots,
                          through_slots=args.through_slots, warm_start=args.warm_start, precision=args.precision)
    clk.stop()
    line = {"metric": "low-rank codec GB/s of fp32 residual input (Algorithm 3 + apply)", "n_gpus": world,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "tf32/f64",
            "data": "synthetic", "e2e": None, **out, "clocks": clk.summary()}
    if args.slots:
        line["roofline"]["traffic"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def quant_extra(args, w, world, rank, clk, steps):
    """One more quantised workload (compress + decompress per step, every
    slot in one grouped launch each), timed like the headline: inputs of a
    few distinct steps resident in HBM and cycled, CUDA events per kernel."""
    import activation_residual_compression_02_b200 as cf

    dev = torch.device("cuda", torch.cuda.current_device())
    shapes = [(w.rows, w.cols)] * w.slots
    ctx = cf.Context(shapes, bits=w.bits, group=w.group)
    st = cf.QuantState(shapes, w.bits, w.group, device=dev)
    nsteps = 4                                # the warmup and three distinct compressed steps, cycled
    streams = [synth.SlotStream(w, s, seed=rank, device=dev) for s in range(w.slots)]
    X = [[None] * w.slots for _ in range(nsteps)]
    for s in range(w.slots):
        for t in range(nsteps):
            X[t][s] = streams[s].next().reshape(-1)
        streams[s].state = None
    del streams
    arrs = [ctx._slots(st.slots(X[t])) for t in range(nsteps)]
    L, h = cf.lib(), ctx.handle
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    def step(i, ev=None):
        arr = arrs[0] if i == 0 else arrs[1 + (i - 1) % (nsteps - 1)]
        if ev:
            ev[0].record(stream)
        if L.cf_compress(h, arr, i, sh) != 0:
            raise RuntimeError(L.cf_last_error(h).decode())
        if ev:
            ev[1].record(stream)
        if L.cf_decompress(h, arr, i, sh) != 0:
            raise RuntimeError(L.cf_last_error(h).decode())
        if ev:
            ev[2].record(stream)

    for i in range(args.warmup + 1):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Timed(clk):
        t0.record(stream)
        for k in range(steps):
            step(args.warmup + 1 + k, ev[k])
        t1.record(stream)
        torch.cuda.synchronize()
    if ctx.check() != 0:
        raise RuntimeError(f"device status in the {w.name} run")
    ms = max_over_ranks(t0.elapsed_time(t1), world) / steps
    c_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / steps, world)
    d_ms = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in ev) / steps, world)
    bc, bd = alg_bytes_per_elem(w.bits, w.group)
    peak, _ = hbm_peak()
    n = w.elems
    pair = (bc + bd) * n / (ms * 1e-3) / 1e9
    out = {"metric": METRIC, "value": world * n * 2 / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms,
           "steps": steps, "warmup": args.warmup, "config": workload_config(w),
           "compress": {"ms_per_launch": c_ms, "frac": bc * n / (c_ms * 1e-3) / 1e9 / peak,
                        "alg_bytes_per_launch": bc * n},
           "decompress": {"ms_per_launch": d_ms, "frac": bd * n / (d_ms * 1e-3) / 1e9 / peak,
                          "alg_bytes_per_launch": bd * n},
           "roofline_step": {"achieved": pair, "frac": pair / peak, "frac_of_8tbs": pair / 8000.0,
                             "alg_bytes_per_step": (bc + bd) * n},
           "gpu_launches": 2 * steps, "payload": payload_summary(ctx, w)}
    ctx.close()
    del X, arrs, st
    torch.cuda.empty_cache()
    return out


def run_exchange_bench(args, w):
    """Algorithm 1's K/V all-gather with compressed payloads (PatchAllGather)
    against the same all-gather of the bf16 activations, on N GPUs.  Each rank
    owns the workload's slots as its shard.  At N = 1 the rank decodes its own
    payload (include_self) so that every stage of the step runs."""
    import datetime

    import torch.distributed as dist

    world, rank, local = dist_init()
    if world == 1:
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{29400 + os.getpid() % 500}", rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=120))
    from activation_residual_compression_02_b200.exchange import PatchAllGather, gather_payloads

    dev = torch.device("cuda", torch.cuda.current_device())
    shapes = [(w.rows, w.cols)] * w.slots
    # one bucket at N = 1, where there is no transfer to overlap (1: 0.754 ms, 4: 0.820 ms per FLUX step)
    buckets = args.buckets if args.buckets else (1 if world == 1 else 4)
    ex = PatchAllGather(shapes, bits=w.bits, group=w.group, buckets=buckets, include_self=world == 1)
    nsteps = min(w.steps, 1 + args.warmup + args.steps)
    streams = [synth.SlotStream(w, s, seed=rank, device=dev) for s in range(w.slots)]
    X = [[streams[s].next().reshape(-1) for s in range(w.slots)] for _ in range(nsteps)]
    del streams
    x_bytes = w.elems * 2
    stream = torch.cuda.current_stream()

    def x_at(i):
        return X[1 + (i - 1) % (nsteps - 1)] if nsteps > 1 else X[0]

    ex.step(0, X[0])
    for i in range(1, args.warmup + 1):
        ex.step(i, x_at(i))
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for k in range(args.steps):
            i = args.warmup + 1 + k
            ex.step(i, x_at(i))
        e1.record(stream)
        torch.cuda.synchronize()
    if ex.check() != 0:
        raise RuntimeError("device status in the exchange run")
    ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
    # the same all-gather of the bf16 activations themselves
    flat = torch.cat([x.view(torch.uint8) for x in X[0]])
    for _ in range(args.warmup):
        gather_payloads(flat, world)
    torch.cuda.synchronize()
    barrier(world)
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    for _ in range(args.steps):
        gather_payloads(flat, world)
    r1.record(stream)
    torch.cuda.synchronize()
    raw_ms = max_over_ranks(r0.elapsed_time(r1), world) / args.steps
    pay = sum(b.nbytes for b in ex.send_buf)
    line = {
        "metric": "compressed K/V all-gather step (compress + all-gather + decompress), GB/s of bf16 activations",
        "value": world * x_bytes / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{w.name}: {w.slots} slots x {w.rows} x {w.cols} bf16 per rank, k={w.bits}, "
                               f"G={w.group}, patch-parallel all-gather (Algorithm 1), {len(ex.buckets)} buckets",
                   "decoded_peers": len(ex.peers)},
        "payload_bytes_per_rank": pay, "raw_bytes_per_rank": x_bytes,
        "raw_bf16_allgather_ms": raw_ms,
        "note": "raw_bf16_allgather_ms: NCCL all-gather of the same activations uncompressed; at N = 1 both "
                "collectives are local copies",
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del ex
    dist.destroy_process_group()
    return 0


# The exponential unit bounds attention with heads of 64: one 2^x per score
# against 4 * 64 flops of the two products.  A microbenchmark of the softmax
# loop (registers only) measured 8.7 cycles per warp-wide ex2 on one
# sub-partition, with one warp or two; at 4 sub-partitions x 148 SMs and the
# 1965 MHz clock that is 4.28e12 exponentials/s, i.e. 1095 TFLOP/s of attention.
XU_CLK_PER_WARP_EX2 = 8.7


def xu_bound_tflops(head_dim=64, sm_mhz=1965.0, sms=148):
    ex2_per_s = sms * 4 * 32 / XU_CLK_PER_WARP_EX2 * sm_mhz * 1e6
    return ex2_per_s * 4 * head_dim / 1e12


def attention_measure(args, w, world, rank, clk, steps):
    """The consumer of the compressed K/V exchange (Algorithms 1 and 2): one
    step of attention over a received shard for every layer of the workload
    (the layer's K and V slots, 4444 tokens x 1920 channels = 30 heads of 64
    for the CogVideoX-shaped shard), three ways:
      recon       cf_decompress of every K/V slot writing bf16(C) in the same
                  pass, then cf_attention on those bf16 tensors;
      cast        cf_decompress, a separate torch cast of each cache to bf16,
                  then cf_attention;
      dequantise  cf_attention reading the caches and the step's payload,
                  dequantising on load and writing the new caches (no
                  decompress launch).
    Returns ms per step of each and the attention kernel's TFLOP/s against
    the measured bf16 peak and the exponential-unit bound."""
    import activation_residual_compression_02_b200 as cf

    dev = torch.device("cuda", torch.cuda.current_device())
    layers = w.slots
    shapes = [(w.rows, w.cols)] * (2 * layers)        # K and V of every layer
    ctx = cf.Context(shapes, bits=w.bits, group=w.group)
    st = cf.QuantState(shapes, w.bits, w.group, device=dev, recon=True)
    streams = [synth.SlotStream(w, s_, seed=rank, device=dev) for s_ in range(2 * layers)]
    x0 = [s_.next().reshape(-1) for s_ in streams]
    sl = st.slots(x0)
    ctx.compress(sl, 0)
    ctx.decompress(sl, 0)
    del x0
    x1 = [s_.next().reshape(-1) for s_ in streams]
    del streams
    sl = st.slots(x1)
    ctx.compress(sl, 1)                                 # the step's payload
    before = st.cache_all.clone()                       # the receiver's caches before the step
    c_before = [before[c.storage_offset() - st.cache_all.storage_offset():][:c.numel()] for c in st.cache]
    new_all = torch.empty_like(st.cache_all)
    c_new = [new_all[c.storage_offset() - st.cache_all.storage_offset():][:c.numel()] for c in st.cache]
    cast_all = torch.empty(st.cache_all.numel(), dtype=torch.bfloat16, device=dev)
    c_cast = [cast_all[c.storage_offset() - st.cache_all.storage_offset():][:c.numel()] for c in st.cache]
    gq = torch.Generator(device=dev)
    gq.manual_seed(synth.mix_seed(rank, 99))
    q = [torch.randn(w.rows, w.cols, generator=gq, device=dev).to(torch.bfloat16) for _ in range(layers)]
    out = [torch.empty(w.rows, w.cols, dtype=torch.bfloat16, device=dev) for _ in range(layers)]
    rc_slots = ctx._slots(sl)
    plain = st.slots(x1)
    for sl_ in plain:
        sl_.recon = None
    plain_slots = ctx._slots(plain)
    L, h = cf.lib(), ctx.handle
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    def decompress(arr):
        if L.cf_decompress(h, arr, 1, sh) != 0:
            raise RuntimeError(L.cf_last_error(h).decode())

    def attn_bf16(kv_k, kv_v):
        for l_ in range(layers):
            ctx.attention(q[l_], cf.KV(bf16=kv_k[l_]), cf.KV(bf16=kv_v[l_]), out[l_], stream=stream)

    def path_recon():
        decompress(rc_slots)
        attn_bf16(st.recon[0::2], st.recon[1::2])

    def path_cast():
        decompress(plain_slots)
        cast_all.copy_(st.cache_all)
        attn_bf16(c_cast[0::2], c_cast[1::2])

    def path_dequantise():
        for l_ in range(layers):
            kv = [cf.KV(cache_in=c_before[2 * l_ + i], cache_out=c_new[2 * l_ + i], codes=st.codes[2 * l_ + i],
                        scales=st.scales[2 * l_ + i]) for i in range(2)]
            ctx.attention(q[l_], kv[0], kv[1], out[l_], stream=stream)

    def attention_only():
        attn_bf16(st.recon[0::2], st.recon[1::2])

    def time_it(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with Timed(clk):
            e0.record(stream)
            for _ in range(steps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), world) / steps

    ms = {name: time_it(fn) for name, fn in (("attention_only", attention_only), ("recon", path_recon),
                                             ("cast", path_cast), ("dequantise", path_dequantise))}
    if ctx.check() != 0:
        raise RuntimeError("device status in the attention run")
    flops = 4.0 * w.rows * w.rows * w.cols * layers     # Q K^T and P V: 2 * 2 * lq * lk * 64 per head
    peak = bf16_peak()
    tf = flops / (ms["attention_only"] * 1e-3) / 1e12
    xu = xu_bound_tflops()
    ctx.close()
    return {
        "workload": f"{w.name}: {layers} layers, K and V slots of {w.rows} tokens x {w.cols} channels "
                    f"({w.cols // 64} heads of 64), k={w.bits}, G={w.group}; queries {w.rows} x {w.cols}",
        "steps": steps, "paths_ms": ms, "ms_per_step": ms["recon"],
        "roofline": {"bound": "tensor", "kernel": "k_attention<bf16>", "achieved": tf, "peak": peak[0],
                     "peak_kind": peak[1], "unit": "TFLOP/s", "frac": tf / peak[0],
                     "traffic": recorded_traffic("attention", "cf_attention.cu"),
                     "tensor_pipe": recorded_traffic("attention", "cf_attention.cu", "tensor_pipe_active"),
                     "xu_pipe": recorded_traffic("attention", "cf_attention.cu", "xu_pipe_active"),
                     "flops_per_step": flops, "xu_bound": xu, "frac_of_xu_bound": tf / xu,
                     "xu_bound_how": "4 sub-partitions x 148 SMs x 32 lanes / 8.7 cycles per warp-wide ex2 "
                                     "(measured) x 1965 MHz x 256 flops per exponential (heads of 64)"},
        "dequantise_vs_recon": ms["dequantise"] / ms["recon"],
        "note": "recon: cf_decompress writing bf16(C) in its pass + cf_attention on bf16; cast: cf_decompress + "
                "torch cast of each cache + cf_attention; dequantise: cf_attention reading C_{t-1}, codes and scales "
                "and writing C_t (no decompress launch)",
        "gpu_launches_per_step": {"attention_only": layers, "recon": 1 + layers, "cast": 1 + layers,
                                  "dequantise": layers},
    }


def run_attention_bench(args, w):
    """`--attention`: the attention measurement as the headline of its own line."""
    world, rank, local = dist_init()
    clk = ClockSampler(torch.cuda.current_device()).start()
    r = attention_measure(args, w, world, rank, clk, args.steps)
    clk.stop()
    line = {
        "metric": "attention step over a received K/V shard (every layer, recon path): ms per step",
        "value": r["ms_per_step"], "unit": "ms", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": r["ms_per_step"], "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": r["workload"], "l2": "inputs larger than L2 (every layer's caches, payloads and "
                                                     "queries)"},
        "paths_ms": r["paths_ms"], "roofline": r["roofline"], "dequantise_vs_recon": r["dequantise_vs_recon"],
        "note": r["note"], "gpu_launches": args.steps * r["gpu_launches_per_step"]["recon"],
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cf", "reference"], default="cf")
    ap.add_argument("--workload", default="flux", choices=["flux", "cogvideox", "stress", "tiny", "lowrank"])
    ap.add_argument("--cpu-steps", type=int, default=8)
    ap.add_argument("--slots", type=int, default=None, help="override the slot count (profiling a smaller case)")
    ap.add_argument("--budget", type=float, default=120.0, help="seconds of oracle work for --impl reference")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-loopback", action="store_true")
    ap.add_argument("--no-lean", action="store_true")
    ap.add_argument("--no-recon", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the CogVideoX-shaped, stress and low-rank extra keys of the default line")
    ap.add_argument("--warm-start", action="store_true", help="low-rank: T = 1 from the previous call's V")
    ap.add_argument("--precision", type=int, default=0, choices=[0, 1, 2],
                    help="low-rank products: 0 automatic, 1 TF32, 2 split (3xTF32)")
    ap.add_argument("--through-slots", action="store_true",
                    help="low-rank: also time cf_compress / cf_decompress in low-rank mode on bf16 slots")
    ap.add_argument("--attention", action="store_true",
                    help="time attention over the received K/V of every layer: recon, cast and dequantise-on-load")
    ap.add_argument("--exchange", action="store_true",
                    help="time the compressed K/V all-gather of patch parallelism instead of the codec alone")
    ap.add_argument("--buckets", type=int, default=None,
                    help="--exchange: slot buckets overlapped with the collective (default 1 at N = 1, else 4)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = synth.WORKLOADS[args.workload]
    if args.slots:
        w = w.scaled(slots=args.slots)
    if args.impl == "reference":
        return run_reference(args, w)
    if w.mode == 1:
        return run_lowrank_bench(args, w)
    if args.exchange:
        return run_exchange_bench(args, w)
    if args.attention:
        return run_attention_bench(args, w if args.workload != "flux" else synth.COGVIDEOX)
    return run_cf(args, w)


if __name__ == "__main__":
    sys.exit(main())
