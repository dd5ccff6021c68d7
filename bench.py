"""Benchmark of the routed sigmoid top-k MoE FFN layer on B200.

Step = one pass of the hot path over one batch of the ``prefill`` workload
(m=4096 tokens, hidden 4096, expert intermediate 1536, 256 experts, top-8):
sigmoid + selection-bias routing from the logits, expert map, gate/up grouped
GEMM with fused SwiGLU, down grouped GEMM with the weighted scatter, ordered
combine.  The same run times, each with its own step, stage split, roofline,
end-to-end figure and CPU baseline, the two tensor-bound layers: ``skewed``
(the prefill layer with every token forced onto experts 0..7) and ``long``
(m=16384, hidden 2048, inter 768, 128 experts, top-8, slotted input rows);
and the decode-shaped matmul by expert id (m=8, k=4096, n=1536, 256 experts,
top-8; the weight-streaming path) under ``decode``.

``value`` is routed-expert TFLOP/s summed over ranks (2*m*top_k*3*hidden*inter
per step); ``tokens_per_s`` is m per step.  Inputs are resident in HBM when the
timed region starts; the expert weights (9.7 GB) are larger than L2, so every
step streams them from HBM.  ``e2e`` repeats the measurement through the same
public API with the step's inputs (x, logits) copied from pinned host memory
and the output y copied back, inside the timed region.

``--impl reference`` times the CPU oracle (f64) on the host cores on a bounded
sample of tokens per step instead (rank 0 only).

Launch: ``python bench.py [--gpus N --steps K --warmup W]``; for N > 1 under
``torch.distributed.run`` each rank runs an independent replica (the layer
shards by tokens with no exchange step: weak scaling, no collective on the
data path; NCCL is used only for the barrier and the max over ranks).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import moe_inputs  # noqa: E402

METRIC = "routed-expert TFLOP/s (prefill) & HBM GB/s (decode), tokens/s per MoE layer"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self._t:
            self._t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- workload
def prefill_flops(cfg) -> float:
    return 2.0 * cfg.m * cfg.top_k * 3.0 * cfg.hidden * cfg.inter


def gate_up_flops(cfg) -> float:
    return 2.0 * cfg.m * cfg.top_k * cfg.hidden * 2.0 * cfg.inter


def down_flops(cfg) -> float:
    return 2.0 * cfg.m * cfg.top_k * cfg.inter * cfg.hidden


def gate_up_bytes(cfg, n_active: int) -> float:
    """Algorithmic HBM bytes of one gate/up launch: the W_gate and W_up rows of
    every expert with routed rows, x read once, the 16-bit activation written
    once."""
    rows = cfg.m * cfg.top_k
    x_rows = cfg.m if cfg.layout == 0 else rows
    return (n_active * 2.0 * cfg.inter * cfg.hidden * 2 + x_rows * cfg.hidden * 2
            + rows * cfg.inter * 2.0)


def down_bytes(cfg, n_active: int) -> float:
    """W_down of every expert with rows, the 16-bit activation read once, the
    f32 per-slot rows written once."""
    rows = cfg.m * cfg.top_k
    return n_active * cfg.hidden * cfg.inter * 2.0 + rows * cfg.inter * 2.0 + rows * cfg.hidden * 4.0


def launches_per_step(cfg) -> int:
    """Library kernels one layer step launches: the routing kernel, then
    moe_ffn_forward -- on the grouped path the expert map (one kernel up to
    2048 routed rows, three above), gate/up, the W_down fp16 copy kernel
    (from 512 routed rows), down and the combine; on the streaming path
    (<= 128 routed rows) gate/up with the map inside, down and the combine."""
    rows = cfg.m * cfg.top_k
    if rows <= 128:
        return 1 + 3
    return 1 + (1 if rows <= 2048 else 3) + 1 + (1 if rows >= 512 else 0) + 1 + 1


def io_bytes(cfg):
    """Host<->device bytes of one end-to-end step: x and logits in, y out."""
    x_rows = cfg.m if cfg.layout == 0 else cfg.m * cfg.top_k
    return x_rows * cfg.hidden * 2 + cfg.m * cfg.n_experts * 4, cfg.m * cfg.hidden * 4


KERNEL_SOURCE = os.path.join(ROOT, "mixture_experts_routed_sigmoid_b200", "csrc", "grouped_gemm.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gate_up_prefill_traffic.json")


def kernel_source_hash() -> str:
    """Hash of the grouped GEMM's code: its source with // comments, trailing
    blanks and empty lines removed, so that a comment edit keeps the measured
    traffic while any code change voids it."""
    import hashlib
    lines = []
    with open(KERNEL_SOURCE, encoding="utf-8") as f:
        for line in f:
            code = line.split("//", 1)[0].rstrip()
            if code:
                lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


def measured_traffic(workload: str):
    """DRAM bytes per launch of the gate/up kernel from the committed ncu
    summary, or None if the kernel source changed since it was taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        rec = t["gate_up"][workload]
        if t.get("kernel_sha") != kernel_source_hash():
            return None
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        return None


def layer_inputs(cfg, seed: int, device, base=None):
    """Seeded inputs of one FFN layer workload.  ``base``: reuse another
    layer's tensors of the same shape (the skewed layer is the prefill layer
    with forced ids)."""
    if base is not None:
        inp = dict(base)
        inp["ids"] = moe_inputs.skewed_ids(cfg.m, cfg.top_k, device)
        return inp
    return moe_inputs.ffn_inputs(cfg, seed=seed, device=device)


def time_layer(args, cfg, inp, world: int, device, stream, clocks=None):
    """Times K steps of one layer (routing from the logits, or the weights of
    forced ids, then moe_ffn_forward) with CUDA events on the launching
    stream, then the same step end to end from pinned host buffers."""
    import mixture_experts_routed_sigmoid_b200 as moe

    logits, bias, x = inp["logits"], inp["bias"], inp["x"]
    Wg, Wu, Wd = inp["W_gate"], inp["W_up"], inp["W_down"]
    forced = inp.get("ids")
    m, top_k = cfg.m, cfg.top_k
    ids = torch.empty((m, top_k), dtype=torch.int32, device=device)
    w = torch.empty((m, top_k), dtype=torch.float32, device=device)
    y = torch.empty((m, cfg.hidden), dtype=torch.float32, device=device)
    ws = torch.empty(moe.moe_ffn_workspace(m, cfg.hidden, cfg.inter, top_k, cfg.n_experts),
                     dtype=torch.uint8, device=device)
    if forced is not None:
        ids.copy_(forced)

    def route(lg):
        if forced is None:
            moe.moe_route_topk(lg, bias, top_k, ids=ids, weights=w)
        else:
            moe.moe_route_weights(lg, ids, weights=w)

    def step(begin=None):
        if begin is not None:
            begin.record(stream)
        route(logits)
        moe.moe_ffn_forward(x, ids, w, Wg, Wu, Wd, layout=cfg.layout, y=y, ws=ws)

    n_stage = 5
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_stage)] for _ in range(args.steps)]
    ev_begin = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]

    for _ in range(args.warmup):
        step()
    for evs in ev:
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize()
    n_active = int((torch.bincount(ids.view(-1).long(), minlength=cfg.n_experts) > 0).sum())

    # ------------------------------------------------ timed region (device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.start()
        time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    # SM cycle counters and the ns timer read on the GPU right before and
    # after the timed steps: the region's exact average SM clock
    n_probe = 2 * torch.cuda.get_device_properties(device).multi_processor_count
    probe = [torch.zeros((n_probe, 3), dtype=torch.int64, device=device) for _ in range(2)]
    moe.moe_clock_probe(probe[0])
    t0.record(stream)
    for i in range(args.steps):
        moe.moe_set_stage_events(ev[i], prerecord=False)
        step(ev_begin[i])
    moe.moe_set_stage_events(None)
    t1.record(stream)
    moe.moe_clock_probe(probe[1])
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = t0.elapsed_time(t1) / args.steps
    mhz = moe.probe_clock_mhz(probe[0], probe[1])
    region_clocks = None if mhz is None else {"sm_mhz_avg": mhz, "source": "SM cycle counter / "
                                              "global ns timer over the timed steps"}
    # stages: route, expert map, gate/up, down, combine (mean over steps)
    stage_ms = [sum(ev_begin[i].elapsed_time(ev[i][0]) for i in range(args.steps)) / args.steps]
    stage_ms += [sum(ev[i][s].elapsed_time(ev[i][s + 1]) for i in range(args.steps)) / args.steps
                 for s in range(n_stage - 1)]
    per_step = sorted(ev_begin[i].elapsed_time(ev[i][n_stage - 1]) for i in range(args.steps))
    quant = {q: per_step[min(len(per_step) - 1, int(round(f * (len(per_step) - 1))))]
             for q, f in (("p25", 0.25), ("p50", 0.5), ("p75", 0.75))}

    # ------------------------------------------------ e2e through host buffers
    # Every step copies its own x and logits in from pinned host memory and
    # its y back out.  Copies run on their own streams, double-buffered, so
    # the copies of step i+1 / i-1 overlap the kernels of step i.
    n_buf = 2
    x_host = [x.cpu().pin_memory() for _ in range(n_buf)]
    lg_host = [logits.cpu().pin_memory() for _ in range(n_buf)]
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(n_buf)]
    x_dev = [torch.empty_like(x) for _ in range(n_buf)]
    lg_dev = [torch.empty_like(logits) for _ in range(n_buf)]
    y_dev = [torch.empty_like(y) for _ in range(n_buf)]
    s_in = torch.cuda.Stream(device)
    s_out = torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(n_buf)]
    ev_comp = [torch.cuda.Event() for _ in range(n_buf)]
    ev_out = [torch.cuda.Event() for _ in range(n_buf)]
    for b in range(n_buf):  # all buffers start free
        ev_comp[b].record(stream)
        ev_out[b].record(stream)

    def e2e_step(i):
        b = i % n_buf
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_comp[b])          # kernels of step i-2 done reading buffer b
            x_dev[b].copy_(x_host[b], non_blocking=True)
            lg_dev[b].copy_(lg_host[b], non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])              # y[b] of step i-2 copied out
        route(lg_dev[b])
        moe.moe_ffn_forward(x_dev[b], ids, w, Wg, Wu, Wd, layout=cfg.layout, y=y_dev[b], ws=ws)
        ev_comp[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            y_host[b].copy_(y_dev[b], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    if not torch.equal(y_host[(args.steps - 1) % n_buf].to(device), y_dev[(args.steps - 1) % n_buf]):
        raise RuntimeError("end-to-end output copy does not match the device result")
    return {"ms": ms, "stage_ms": stage_ms, "step_quantiles": quant, "e2e_ms": e2e_ms,
            "n_active": n_active, "region_clocks": region_clocks}


def run_gpu(args, cfg, rank: int, world: int, device: torch.device):
    """The headline layer, then (for the prefill headline) the skewed and long
    layers, the decode matmul by expert id, the decode-size layer and the
    router projection.  Clocks are sampled across the layers' timed steps
    (the nvidia-smi poller is stopped before the short decode-size calls,
    whose eager launches it would otherwise delay)."""
    peaks = load_peaks()
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    clocks = ClockSampler(device.index if device.index is not None else 0)
    inp = layer_inputs(cfg, args.seed + rank, device)
    res = time_layer(args, cfg, inp, world, device, stream, clocks=clocks)
    res["peaks"] = peaks
    res["layers"] = {}
    if cfg.name == "prefill" and not args.no_extra_layers:
        sk = moe_inputs.SKEWED
        res["layers"]["skewed"] = time_layer(args, sk, layer_inputs(sk, 0, device, base=inp),
                                             world, device, stream)
        del inp
        lg = moe_inputs.LONG
        res["layers"]["long"] = time_layer(args, lg, layer_inputs(lg, args.seed + rank, device),
                                           world, device, stream)
    else:
        del inp
    torch.cuda.empty_cache()
    res["clocks"] = clocks.stop()  # sampled across the layer timings above

    # ------------------------------------------------ decode: weight streaming
    res["decode"] = None if args.no_decode else run_decode(args, rank, device, stream)
    res["tiny"] = None if args.no_decode else run_tiny(args, rank, device, stream)
    res["ep"] = (run_ep_one_rank(args, rank, device, stream)
                 if cfg.name == "prefill" and not args.no_extra_layers else None)
    res["decode_ffn"] = None if args.no_decode else run_decode_ffn(args, rank, device, stream)
    res["router"] = None if args.no_decode else run_router(args, rank, device, stream)
    return res


def run_decode(args, rank, device, stream):
    """Decode-shaped matmul by expert id (weight-streaming path), timed per call
    and per kernel (stage events around the streaming kernel)."""
    import mixture_experts_routed_sigmoid_b200 as moe

    dcfg = moe_inputs.DECODE
    dinp = moe_inputs.matmul_id_inputs(dcfg, seed=args.seed + rank, device=device)
    dy = torch.empty((dcfg.m, dcfg.top_k, dcfg.n), dtype=torch.float32, device=device)
    dws = torch.empty(moe.moe_matmul_id_workspace(dcfg.m, dcfg.n, dcfg.k, dcfg.top_k,
                                                  dcfg.n_experts), dtype=torch.uint8,
                      device=device)
    d_steps = max(args.steps * 10, 50)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(d_steps)]
    for _ in range(max(args.warmup, 3)):
        moe.moe_matmul_id(dinp["x"], dinp["ids"], dinp["W"], y=dy, ws=dws)
    for e3 in evs:
        for e in e3:
            e.record(stream)
    torch.cuda.synchronize()
    d0 = torch.cuda.Event(enable_timing=True)
    d1 = torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for i in range(d_steps):
        moe.moe_set_stage_events(evs[i], prerecord=False)
        moe.moe_matmul_id(dinp["x"], dinp["ids"], dinp["W"], y=dy, ws=dws)
    moe.moe_set_stage_events(None)
    d1.record(stream)
    torch.cuda.synchronize()
    unique = int(torch.unique(dinp["ids"]).numel())
    return {
        "ms": d0.elapsed_time(d1) / d_steps,
        "kernel_ms": sum(evs[i][1].elapsed_time(evs[i][2]) for i in range(d_steps)) / d_steps,
        "map_ms": sum(evs[i][0].elapsed_time(evs[i][1]) for i in range(d_steps)) / d_steps,
        "bytes": (unique * dcfg.n * dcfg.k * 2.0 + dcfg.m * dcfg.k * 2.0
                  + dcfg.m * dcfg.top_k * dcfg.n * 4.0),
        "unique": unique,
    }


def run_ep_one_rank(args, rank, device, stream):
    """The expert-parallel step of the prefill layer at one rank (the
    exchange is a device copy): dispatch (owner sort + row pack), the owner's
    experts (moe_ffn_slots on the packed rows), the combine -- each timed with
    CUDA events, and the output compared bit for bit with moe_ffn_forward."""
    import mixture_experts_routed_sigmoid_b200 as moe
    from mixture_experts_routed_sigmoid_b200.ep import CudaEpOps, SelfComm

    cfg = moe_inputs.PREFILL
    inp = moe_inputs.ffn_inputs(cfg, seed=args.seed + rank, device=device)
    ids, w = moe.moe_route_topk(inp["logits"], inp["bias"], cfg.top_k)
    W = (inp["W_gate"], inp["W_up"], inp["W_down"])
    ops, comm = CudaEpOps(), SelfComm()
    rows = cfg.m * cfg.top_k
    recv_x = torch.empty((rows, cfg.hidden), dtype=torch.bfloat16, device=device)
    recv_e = torch.empty(rows, dtype=torch.int32, device=device)
    d_back = torch.empty((rows, cfg.hidden), dtype=torch.float32, device=device)
    send_x = torch.empty_like(recv_x)
    send_e = torch.empty_like(recv_e)
    counts = torch.empty(1, dtype=torch.int32, device=device)
    ws = torch.empty(moe.moe_ep_dispatch_workspace(cfg.m, cfg.top_k, 1), dtype=torch.uint8,
                     device=device)
    fws = torch.empty(moe.moe_ffn_workspace(rows, cfg.hidden, cfg.inter, 1, cfg.n_experts,
                                            moe.SLOTTED), dtype=torch.uint8, device=device)
    y = torch.empty((cfg.m, cfg.hidden), dtype=torch.float32, device=device)

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        moe.moe_ep_dispatch(inp["x"], ids, cfg.n_experts, 1, send_x=send_x, send_expert=send_e,
                            send_counts=counts, ws=ws)
        mark(1)
        comm.all_to_all(recv_x, send_x, [rows], [rows])
        comm.all_to_all(recv_e, send_e, [rows], [rows])
        mark(2)
        moe.moe_ffn_slots(recv_x.view(rows, 1, cfg.hidden), recv_e.view(rows, 1), *W,
                          layout=moe.SLOTTED, d_slots=d_back.view(rows, 1, cfg.hidden), ws=fws)
        mark(3)
        moe.moe_ep_combine(d_back, w, 1, ws, y=y)
        mark(4)

    for _ in range(max(args.warmup, 3)):
        step()
    n = max(args.steps, 10)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n)]
    torch.cuda.synchronize()
    for i in range(n):
        step(evs[i])
    torch.cuda.synchronize()
    part = [sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(n)) / n for j in range(4)]
    y_ref = moe.moe_ffn_forward(inp["x"], ids, w, *W)
    torch.cuda.synchronize()
    same = bool(torch.equal(y.view(torch.int32), y_ref.view(torch.int32)))
    pack_bytes = 2.0 * rows * cfg.hidden * 2          # rows read, packed rows written
    comb_bytes = rows * cfg.hidden * 4.0 + cfg.m * cfg.hidden * 4.0
    return {"dispatch_ms": part[0], "exchange_ms": part[1], "experts_ms": part[2],
            "combine_ms": part[3], "dispatch_bytes": pack_bytes, "combine_bytes": comb_bytes,
            "bits_equal_moe_ffn_forward": same}


def run_tiny(args, rank, device, stream):
    """The tiny matmul by expert id (m=4, k=64, n=32, 8 experts, top-2): a
    launch-latency-bound call, timed per call over many back-to-back calls."""
    import mixture_experts_routed_sigmoid_b200 as moe

    cfg = moe_inputs.TINY
    inp = moe_inputs.matmul_id_inputs(cfg, seed=args.seed + rank, device=device)
    y = torch.empty((cfg.m, cfg.top_k, cfg.n), dtype=torch.float32, device=device)
    ws = torch.empty(moe.moe_matmul_id_workspace(cfg.m, cfg.n, cfg.k, cfg.top_k, cfg.n_experts),
                     dtype=torch.uint8, device=device)
    for _ in range(max(args.warmup, 3)):
        moe.moe_matmul_id(inp["x"], inp["ids"], inp["W"], y=y, ws=ws)
    n = 200
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        moe.moe_matmul_id(inp["x"], inp["ids"], inp["W"], y=y, ws=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    return {"ms": e0.elapsed_time(e1) / n, "m": cfg.m, "n": cfg.n, "k": cfg.k,
            "n_experts": cfg.n_experts, "top_k": cfg.top_k}


def cpu_baseline_matmul_id(cfg, repeats: int = 1):
    """The oracle's matmul by expert id on a whole workload (m tokens), on the
    host cores: wall seconds per call."""
    import oracle

    inp = moe_inputs.matmul_id_inputs(cfg, seed=0, device="cpu")
    xb, Wb = moe_inputs.bf16_bits(inp["x"]), moe_inputs.bf16_bits(inp["W"])
    ids = inp["ids"].numpy()
    oracle.matmul_id(xb, ids, Wb, cfg.layout)  # warm (library load, pages)
    t0 = time.perf_counter()
    for _ in range(repeats):
        oracle.matmul_id(xb, ids, Wb, cfg.layout)
    dt = (time.perf_counter() - t0) / repeats
    cores = os.cpu_count() or 1
    return {"value": dt * 1e3, "unit": "ms per call", "cores": int(os.environ.get("OMP_NUM_THREADS", cores)),
            "kind": "oracle", "sample": f"the whole {cfg.name} workload (m={cfg.m}), f64 C oracle, "
                                        f"{repeats} call(s)"}


def run_decode_ffn(args, rank, device, stream, m: int = 8):
    """Decode-size MoE layer step on the prefill layer's weights: routing from
    logits + moe_ffn_forward at m tokens (the weight-streaming FFN path)."""
    import mixture_experts_routed_sigmoid_b200 as moe

    cfg = moe_inputs.PREFILL
    inp = moe_inputs.ffn_inputs(cfg, seed=args.seed + rank, device=device, m=m)
    ids = torch.empty((m, cfg.top_k), dtype=torch.int32, device=device)
    w = torch.empty((m, cfg.top_k), dtype=torch.float32, device=device)
    y = torch.empty((m, cfg.hidden), dtype=torch.float32, device=device)
    ws = torch.empty(moe.moe_ffn_workspace(m, cfg.hidden, cfg.inter, cfg.top_k, cfg.n_experts),
                     dtype=torch.uint8, device=device)

    def step():
        moe.moe_route_topk(inp["logits"], inp["bias"], cfg.top_k, ids=ids, weights=w)
        moe.moe_ffn_forward(inp["x"], ids, w, inp["W_gate"], inp["W_up"], inp["W_down"], y=y, ws=ws)

    for _ in range(max(args.warmup, 3)):
        step()
    n = max(args.steps, 20)
    # eager steps as a caller runs them (no stage events)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    # then the same steps with the library's stage events: the two streaming
    # kernels (gate/up + SwiGLU, down + weight) on their own
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n)]
    for e5 in evs:
        for e in e5:
            e.record(stream)
    torch.cuda.synchronize()
    for i in range(n):
        moe.moe_set_stage_events(evs[i], prerecord=False)
        step()
    moe.moe_set_stage_events(None)
    torch.cuda.synchronize()
    kernel_ms = sum(evs[i][1].elapsed_time(evs[i][2]) for i in range(n)) / n
    y_eager = y.clone()

    # the same step captured once in a CUDA graph and replayed (the library
    # call sequence is capturable: no allocation, no host synchronisation)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    if not torch.equal(y.view(torch.int32), y_eager.view(torch.int32)):
        raise RuntimeError("graph replay of the decode-size layer changed the output bits")
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(n):
        graph.replay()
    g1.record(stream)
    torch.cuda.synchronize()
    graph_ms = g0.elapsed_time(g1) / n
    del graph
    unique = int(torch.unique(ids).numel())
    wbytes = unique * 3.0 * cfg.inter * cfg.hidden * 2
    return {"m": m, "ms": ms, "kernel_ms": kernel_ms, "graph_ms": graph_ms,
            "unique_experts": unique, "weight_bytes": wbytes}


def run_router(args, rank, device, stream):
    """Router projection x . W_router^T + routing at the prefill layer's shape."""
    import mixture_experts_routed_sigmoid_b200 as moe

    cfg = moe_inputs.PREFILL
    g = moe_inputs.generator(args.seed + rank + 7, device)
    x = moe_inputs.bf16_normal((cfg.m, cfg.hidden), 1.0, g, device)
    Wr = moe_inputs.bf16_normal((cfg.n_experts, cfg.hidden), 0.02, g, device)
    bias = moe_inputs.uniform_bias(cfg.n_experts, 0.1, g, device)
    logits = torch.empty((cfg.m, cfg.n_experts), dtype=torch.float32, device=device)
    ids = torch.empty((cfg.m, cfg.top_k), dtype=torch.int32, device=device)
    w = torch.empty((cfg.m, cfg.top_k), dtype=torch.float32, device=device)
    ws = torch.empty(moe.moe_router_workspace(cfg.m, cfg.hidden, cfg.n_experts), dtype=torch.uint8,
                     device=device)
    for _ in range(max(args.warmup, 3)):
        moe.moe_router_topk(x, Wr, bias, cfg.top_k, logits=logits, ids=ids, weights=w, ws=ws)
    torch.cuda.synchronize()
    n = max(args.steps, 20)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        moe.moe_router_topk(x, Wr, bias, cfg.top_k, logits=logits, ids=ids, weights=w, ws=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    # algorithmic bytes: x and W_router read once, logits, ids and weights written once
    nbytes = (cfg.m * cfg.hidden * 2 + cfg.n_experts * cfg.hidden * 2 + cfg.m * cfg.n_experts * 4
              + cfg.m * cfg.top_k * 8)
    return {"m": cfg.m, "hidden": cfg.hidden, "n_experts": cfg.n_experts, "ms": ms,
            "tflops": 2.0 * cfg.m * cfg.hidden * cfg.n_experts / (ms * 1e-3) / 1e12,
            "algorithmic_bytes": float(nbytes), "gbs": nbytes / (ms * 1e-3) / 1e9}


def reduce_max(v: float, world: int, device) -> float:
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def cpu_baseline(cfg=moe_inputs.PREFILL, target_s: float = 12.0):
    """The oracle as it stands, on the host cores, on a bounded token sample of
    one layer workload (its routing for all tokens is cheap and not counted;
    the FFN rows cost 2*top_k*3*hidden*inter f64 FLOPs each)."""
    import numpy as np

    import oracle

    inp = moe_inputs.ffn_inputs(cfg, seed=0, device="cuda" if torch.cuda.is_available() else "cpu")
    logits = inp["logits"].cpu().numpy()
    bias = inp["bias"].cpu().numpy()
    forced = inp.get("ids")
    bits = moe_inputs.bf16_bits
    xb, gb, ub, db = bits(inp["x"]), bits(inp["W_gate"]), bits(inp["W_up"]), bits(inp["W_down"])
    del inp
    if forced is None:
        ids, w, _ = oracle.route(logits, bias, cfg.top_k)
    else:
        ids = forced.cpu().numpy()
        w = oracle.route_weights(logits, ids)
    cores = os.cpu_count() or 1
    n = max(1, min(cores, 64))

    def run(count):
        t0 = time.perf_counter()
        oracle.ffn(xb, ids, w, gb, ub, db, layout=cfg.layout,
                   tokens=np.arange(count, dtype=np.int32))
        return time.perf_counter() - t0

    per_tok = run(n) / n
    n2 = int(max(n, min(cfg.m, target_s / max(per_tok, 1e-6))))
    n2 = max(n, (n2 // n) * n)
    dt = run(n2)
    flops = 2.0 * n2 * cfg.top_k * 3 * cfg.hidden * cfg.inter
    threads = int(os.environ.get("OMP_NUM_THREADS", cores))
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{n2} of {cfg.m} {cfg.name} tokens (routing for all tokens excluded), "
                      f"f64 C oracle, {dt:.1f} s", "tokens_per_s": n2 / dt}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    import numpy as np

    import oracle

    cfg = moe_inputs.PREFILL
    inp = moe_inputs.ffn_inputs(cfg, seed=args.seed, device="cuda" if torch.cuda.is_available() else "cpu")
    logits = inp["logits"].cpu().numpy()
    bias = inp["bias"].cpu().numpy()
    bits = moe_inputs.bf16_bits
    xb, gb, ub, db = bits(inp["x"]), bits(inp["W_gate"]), bits(inp["W_up"]), bits(inp["W_down"])
    del inp
    cores = os.cpu_count() or 1
    tok = max(1, min(cores, 32))  # tokens per step: one per core, bounded
    ids, w, _ = oracle.route(logits, bias, cfg.top_k)

    def step(i):
        sl = np.arange(i * tok, (i + 1) * tok, dtype=np.int32) % cfg.m
        oracle.route(logits[sl], bias, cfg.top_k)
        oracle.ffn(xb, ids, w, gb, ub, db, tokens=sl)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = (time.perf_counter() - t0) / args.steps
    flops = 2.0 * tok * cfg.top_k * 3 * cfg.hidden * cfg.inter
    value = flops / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "prefill", "m": cfg.m, "hidden": cfg.hidden, "inter": cfg.inter,
                   "n_experts": cfg.n_experts, "top_k": cfg.top_k,
                   "sample_tokens_per_step": tok},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{tok} prefill tokens per step (routing + FFN), f64 C oracle"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "tokens_per_s": tok / dt,
    }
    print(json.dumps(line), flush=True)


def stage_dict(stage_ms):
    return {"route": stage_ms[0], "expert_map": stage_ms[1], "gate_up_swiglu": stage_ms[2],
            "down_scatter": stage_ms[3], "combine": stage_ms[4]}


def layer_object(cfg, world: int, r: dict, ms: float, e2e_ms: float, peaks: dict) -> dict:
    """Sub-object of one tensor-bound layer (skewed, long): its step time and
    routed TFLOP/s against both bf16 peaks, the stage split, the gate/up
    kernel's tensor roofline and the end-to-end figure."""
    flops = prefill_flops(cfg)
    tflops = world * flops / (ms * 1e-3) / 1e12
    gu_ms, dn_ms = r["stage_ms"][2], r["stage_ms"][3]
    gu_tf = gate_up_flops(cfg) / (gu_ms * 1e-3) / 1e12
    dn_tf = down_flops(cfg) / (dn_ms * 1e-3) / 1e12
    h2d, d2h = io_bytes(cfg)
    return {
        "workload": cfg.name, "m": cfg.m, "hidden": cfg.hidden, "inter": cfg.inter,
        "n_experts": cfg.n_experts, "top_k": cfg.top_k,
        "layout": "slotted" if cfg.layout else "shared_per_token",
        "routing": ("sigmoid + selection bias" if cfg.routing == "router"
                    else f"{cfg.routing} forced ids"),
        "experts_with_rows": r["n_active"],
        "ms_per_step": ms, "step_ms_quantiles": r["step_quantiles"],
        "TFLOP/s": tflops, "tokens_per_s": world * cfg.m / (ms * 1e-3),
        "frac_of_bf16_burst": tflops / world / peaks["bf16_tflops"],
        "frac_of_bf16_sustained": tflops / world / peaks["bf16_tflops_sustained"],
        "stage_ms": stage_dict(r["stage_ms"]),
        "roofline": {
            "kernel": "grouped_gemm_kernel<0> (gate/up + SwiGLU)", "bound": "tensor",
            "achieved": gu_tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": gu_tf / peaks["bf16_tflops"],
            "frac_of_sustained": gu_tf / peaks["bf16_tflops_sustained"],
            "traffic": None, "peak_source": peaks["source"],
            "algorithmic_flops": gate_up_flops(cfg),
            "down_kernel": {"achieved": dn_tf, "frac": dn_tf / peaks["bf16_tflops"],
                            "algorithmic_flops": down_flops(cfg)},
        },
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "region_clocks": r.get("region_clocks"),
    }


def compose_line(args, cfg, world: int, res: dict, ms: float, e2e_ms: float,
                 layer_times=None) -> dict:
    """The bench JSON line from rank 0's results and the max-over-ranks times
    (ms per step of the device-timed and end-to-end legs; ``layer_times``
    maps each extra layer to its max-over-ranks (ms, e2e_ms))."""
    peaks = res["peaks"]
    flops = prefill_flops(cfg)
    value = world * flops / (ms * 1e-3) / 1e12
    gu_ms = res["stage_ms"][2]
    gu_bytes = gate_up_bytes(cfg, res["n_active"])
    achieved = gu_bytes / (gu_ms * 1e-3) / 1e9
    rows = cfg.m * cfg.top_k
    h2d, d2h = io_bytes(cfg)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": cfg.name, "m": cfg.m, "hidden": cfg.hidden, "inter": cfg.inter,
            "n_experts": cfg.n_experts, "top_k": cfg.top_k,
            "layout": "slotted" if cfg.layout else "shared_per_token",
            "routing": ("sigmoid + selection bias, top-8, weights s/sum(s)"
                        if cfg.routing == "router" else
                        f"{cfg.routing} forced ids, weights s/sum(s)"),
            "accumulate": "f32", "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (%.2f GB of expert weights, %.2f GB of per-step "
                  "activations)" % (3 * cfg.n_experts * cfg.hidden * cfg.inter * 2 / 1e9,
                                    (rows * cfg.hidden * 8 + rows * cfg.inter * 8) / 1e9),
        },
        "tokens_per_s": world * cfg.m / (ms * 1e-3),
        "stage_ms": stage_dict(res["stage_ms"]),
        "step_ms_quantiles": res.get("step_quantiles"),
        "roofline": {
            "kernel": "grouped_gemm_kernel<0> (gate/up + SwiGLU)",
            "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": measured_traffic(cfg.name),
            "peak_source": peaks["source"],
            "algorithmic_bytes": gu_bytes,
            "tensor_frac_of_layer": value / world / peaks["bf16_tflops"],
            "down_kernel": {
                "achieved": down_bytes(cfg, res["n_active"]) / (res["stage_ms"][3] * 1e-3) / 1e9,
                "frac": down_bytes(cfg, res["n_active"]) / (res["stage_ms"][3] * 1e-3) / 1e9
                / peaks["hbm_gbs"],
                "algorithmic_bytes": down_bytes(cfg, res["n_active"])},
        },
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": args.steps * launches_per_step(cfg),
        "clocks": res["clocks"],
        "region_clocks": res.get("region_clocks"),
    }
    layers = res.get("layers") or {}
    for name, r in layers.items():
        lcfg = moe_inputs.CONFIGS[name]
        lms, le2e = (layer_times or {}).get(name, (r["ms"], r["e2e_ms"]))
        line[name] = layer_object(lcfg, world, r, lms, le2e, peaks)
        line["gpu_launches"] += args.steps * launches_per_step(lcfg)
    dec = res["decode"]
    if dec is not None:
        d_gbs = dec["bytes"] / (dec["kernel_ms"] * 1e-3) / 1e9
        line["decode"] = {
            "workload": "decode", "m": 8, "k": 4096, "n": 1536, "n_experts": 256,
            "top_k": 8, "unique_experts": dec["unique"], "ms_per_call": dec["ms"],
            "expert_map_ms": dec["map_ms"], "stream_kernel_ms": dec["kernel_ms"],
            "GB/s": d_gbs, "hbm_frac": d_gbs / peaks["hbm_gbs"],
            "algorithmic_bytes": dec["bytes"],
            "tokens_per_s": 8 / (dec["ms"] * 1e-3)}
    dffn = res.get("decode_ffn")
    if dffn is not None:
        gbs = dffn["weight_bytes"] / (dffn["ms"] * 1e-3) / 1e9
        line["decode_ffn"] = {
            "workload": "prefill layer at m=%d (routing + weight-streaming FFN)" % dffn["m"],
            "ms_per_step": dffn["ms"], "tokens_per_s": dffn["m"] / (dffn["ms"] * 1e-3),
            "unique_experts": dffn["unique_experts"], "weight_GB/s": gbs,
            "hbm_frac": gbs / peaks["hbm_gbs"]}
        if dffn.get("kernel_ms"):
            k_gbs = dffn["weight_bytes"] / (dffn["kernel_ms"] * 1e-3) / 1e9
            line["decode_ffn"]["stream_kernels"] = {
                "ms": dffn["kernel_ms"], "weight_GB/s": k_gbs, "hbm_frac": k_gbs / peaks["hbm_gbs"]}
        if dffn.get("graph_ms"):
            g_gbs = dffn["weight_bytes"] / (dffn["graph_ms"] * 1e-3) / 1e9
            line["decode_ffn"]["cuda_graph"] = {
                "ms_per_step": dffn["graph_ms"],
                "tokens_per_s": dffn["m"] / (dffn["graph_ms"] * 1e-3),
                "weight_GB/s": g_gbs, "hbm_frac": g_gbs / peaks["hbm_gbs"]}
    ep = res.get("ep")
    if ep is not None:
        hbm = peaks["hbm_gbs"]
        d_gbs = ep["dispatch_bytes"] / (ep["dispatch_ms"] * 1e-3) / 1e9
        c_gbs = ep["combine_bytes"] / (ep["combine_ms"] * 1e-3) / 1e9
        line["ep_one_rank"] = {
            "workload": "prefill layer, expert-parallel step at one rank (exchange = device copy)",
            "dispatch_ms": ep["dispatch_ms"], "dispatch_GB/s": d_gbs, "dispatch_hbm_frac": d_gbs / hbm,
            "exchange_copy_ms": ep["exchange_ms"], "owner_experts_ms": ep["experts_ms"],
            "combine_ms": ep["combine_ms"], "combine_GB/s": c_gbs, "combine_hbm_frac": c_gbs / hbm,
            "bits_equal_moe_ffn_forward": ep["bits_equal_moe_ffn_forward"]}
    tiny = res.get("tiny")
    if tiny is not None:
        line["tiny"] = {"workload": "tiny matmul_id (launch-latency bound)", **tiny,
                        "ms_per_call": tiny["ms"]}
    router = res.get("router")
    if router is not None:
        line["router"] = {"workload": "x . W_router^T + routing, m=%d hidden=%d E=%d" % (
            router["m"], router["hidden"], router["n_experts"]), "ms": router["ms"],
            "TFLOP/s": router["tflops"], "algorithmic_bytes": router["algorithmic_bytes"],
            "GB/s": router["gbs"], "hbm_frac": router["gbs"] / peaks["hbm_gbs"]}
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload",
                    choices=["prefill", "skewed", "long", "prefill_e32", "skewed_e8", "long_e16"],
                    default="prefill",
                    help="FFN layer workload of a step (default: prefill)")
    ap.add_argument("--no-extra-layers", action="store_true",
                    help="with the prefill workload, skip the skewed and long layer lines")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode measurement")
    ap.add_argument("--decode-only", action="store_true",
                    help="only the decode matmul_id measurement (for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=300),
            device_id=torch.device("cuda", local))

    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
            return
        device = torch.device("cuda", local)
        if args.decode_only:
            torch.cuda.set_device(device)
            dec = run_decode(args, rank, device, torch.cuda.current_stream(device))
            if rank == 0:
                print(json.dumps({"decode": dec}), flush=True)
            return
        cfg = moe_inputs.CONFIGS[args.workload]
        res = run_gpu(args, cfg, rank, world, device)
        ms = reduce_max(res["ms"], world, device)
        e2e_ms = reduce_max(res["e2e_ms"], world, device)
        # every rank runs the same layers in the same order, so these
        # collectives line up
        layer_times = {name: (reduce_max(r["ms"], world, device),
                              reduce_max(r["e2e_ms"], world, device))
                       for name, r in res["layers"].items()}
        if rank != 0:
            return
        line = compose_line(args, cfg, world, res, ms, e2e_ms, layer_times)
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(cfg)
            for name in res["layers"]:
                line[name]["cpu_baseline"] = cpu_baseline(moe_inputs.CONFIGS[name], target_s=8.0)
            if "decode" in line:
                line["decode"]["cpu_baseline"] = cpu_baseline_matmul_id(moe_inputs.DECODE)
            if "tiny" in line:
                line["tiny"]["cpu_baseline"] = cpu_baseline_matmul_id(moe_inputs.TINY, repeats=100)
        print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
