#!/usr/bin/env python
"""Benchmark of the batched multi-agent decode-and-verify step on B200.

One step = one pass of the whole hot path over one packed batch: 4 agents x
(next token + 2 drafts) = 12 rows through a 64-layer synthetic Q4_K/Q6_K
decoder stack (hidden 5120, intermediate 17408, 48 query / 8 KV heads of 128),
each layer's quantized weights streamed once for all 12 rows, each agent's
rows attending over its own bf16 KV cache. Inputs are synthetic and seeded
(weights, caches and rows drawn in device memory); the step streams ~13.7 GB
of weights, far more than the 126 MB L2, so no L2 flush is needed between
steps.

Metric: decode-step ms and weight-stream GB/s at 12 rows. ``value`` is the
weight-stream rate: quantized weight bytes per step x GPUs / step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle on the host cores

Multi-GPU: replicas only (every GPU holds the whole stack and serves its own
agents; nothing is exchanged between GPUs), launched one process per GPU.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode-step ms and weight-stream GB/s at M=12 vs B200 HBM peak (1 GPU)"
SEED = 20261202

# name -> (description, layers, rows per agent, agents, cached tokens per agent)
WORKLOADS = {
    "stack12_ctx1k": ("64-layer Q4_K stack (hidden 5120, inter 17408, down Q6_K), 12 rows = 4 agents x 3, "
                      "1024 cached tokens per agent", 64, 3, 4, 1024),
    "stack12_ctx23k": ("64-layer Q4_K stack, 12 rows = 4 agents x 3, 23000 cached tokens per agent "
                       "(GQA 48/8 heads, bf16 KV)", 64, 3, 4, 23000),
    "stack12_ctx23k_q8": ("64-layer Q4_K stack, 12 rows = 4 agents x 3, 23000 cached tokens per agent "
                          "(GQA 48/8 heads, q8_0 KV)", 64, 3, 4, 23000),
}
KV_Q8_WORKLOADS = {"stack12_ctx23k_q8"}
for _m in (1, 2, 3, 4, 6, 8, 12, 16):
    WORKLOADS[f"stack_m{_m}"] = (f"64-layer Q4_K stack, {_m} rows (row-count sweep), 1024 cached tokens",
                                 64, _m, 1, 1024)


class Workload:
    """A synthetic stack, its KV caches and one packed batch, all in device memory."""

    def __init__(self, name, device="cuda", seed=SEED, n_layers=None, shape=None, rows_per_agent=None,
                 n_agents=None, ctx=None):
        import quantized_agent_decode_b200 as q
        desc, L, rpa, na, cl = WORKLOADS.get(name, ("custom", 64, 3, 4, 1024))
        self.name, self.desc = name, desc
        self.seed, self.device = seed, device
        L = n_layers or L
        rpa = rows_per_agent or rpa
        na = n_agents or na
        cl = ctx if ctx is not None else cl
        sh = shape or synth.StackShape(n_layers=L)
        sh.n_layers = L
        self.shape, self.rows_per_agent, self.n_agents, self.ctx = sh, rpa, na, cl
        self.M = rpa * na
        self.kv_cap = cl + rpa
        self.kv_q8 = name in KV_Q8_WORKLOADS
        g = synth.torch_gen(seed, device, 0)
        H, I, hd = sh.hidden, sh.inter, sh.head_dim
        nq, nkv = sh.n_qh * hd, sh.n_kvh * hd
        self.w_qkv, self.w_o, self.w_gu, self.w_down, self.kc, self.vc = [], [], [], [], [], []
        for layer in range(L):
            gl = synth.torch_gen(seed, device, synth.layer_weight_tag(layer, 0))
            self.w_qkv.append(torch.cat([synth.q4k_matrix_torch(gl, nq, H, device),
                                         synth.q4k_matrix_torch(gl, nkv, H, device),
                                         synth.q4k_matrix_torch(gl, nkv, H, device)]))
            self.w_o.append(synth.q4k_matrix_torch(gl, H, nq, device))
            self.w_gu.append(torch.cat([synth.q4k_matrix_torch(gl, I, H, device),
                                        synth.q4k_matrix_torch(gl, I, H, device)]))
            self.w_down.append(q.q6k_pack(synth.q6k_matrix_torch(gl, H, I, device), H, I))
            if self.kv_q8:
                for caches in (self.kc, self.vc):
                    buf = torch.empty(q.kv_cache_bytes(q.KV_Q8_0, na, sh.n_kvh, self.kv_cap, hd),
                                      dtype=torch.uint8, device=device)
                    codes, scales = q.q8_cache_planes(buf, na, sh.n_kvh, self.kv_cap, hd)
                    c8, s16 = synth.q8_planes_torch(gl, na * sh.n_kvh * self.kv_cap, hd, device)
                    codes.view(-1, hd).copy_(c8)
                    scales.view(-1, hd // 32).copy_(s16.view(torch.int16))
                    caches.append(buf)
            else:
                self.kc.append(synth.bf16_normal_torch(gl, (na, sh.n_kvh, self.kv_cap, hd), device))
                self.vc.append(synth.bf16_normal_torch(gl, (na, sh.n_kvh, self.kv_cap, hd), device))
        self.model = q.Model(hidden=H, inter=I, n_qh=sh.n_qh, n_kvh=sh.n_kvh, head_dim=hd, max_agents=na,
                             kv_cap=self.kv_cap, w_qkv=self.w_qkv, w_o=self.w_o, w_gu=self.w_gu,
                             w_down=self.w_down, k_cache=self.kc, v_cache=self.vc,
                             kv_format=q.KV_Q8_0 if self.kv_q8 else q.KV_BF16)
        self.X = synth.bf16_normal_torch(g, (self.M, H), device)
        self.ars = torch.arange(0, self.M + 1, rpa, dtype=torch.int32, device=device)
        self.lens = torch.full((na,), cl, dtype=torch.int32, device=device)
        self.H_out = torch.empty(self.M, H, dtype=torch.float32, device=device)
        self.ws = q.alloc_ws(self.model.ws_bytes(self.M), device)
        # quantized weight bytes streamed per step: the GGUF blocks of the listed matrices (144 B per Q4_K
        # block, 210 B per Q6_K block); the d-plane row padding of the packed down projection is not counted
        self.weight_bytes = sh.weight_bytes_per_layer() * L
        # keys and values read per step (incl. new rows): bf16, or q8_0 codes + one fp16 scale per 32
        self.kv_bytes = 2 * L * na * sh.n_kvh * (cl + rpa) * (hd + hd // 16 if self.kv_q8 else hd * 2)
        self.act_bytes = L * self.M * (2 * H * 4 + 2 * I * 4 + (nq + 2 * nkv) * 4)  # fp32 outputs/residual

    def down_gguf(self, layer):
        """The GGUF-layout bytes of a layer's down projection, redrawn from its seed."""
        sh = self.shape
        H, I, hd = sh.hidden, sh.inter, sh.head_dim
        nq, nkv = sh.n_qh * hd, sh.n_kvh * hd
        gl = synth.torch_gen(self.seed, self.device, synth.layer_weight_tag(layer, 0))
        for n, k in ((nq, H), (nkv, H), (nkv, H), (H, nq), (I, H), (I, H)):  # same draw order as __init__
            synth.q4k_matrix_torch(gl, n, k, self.device)
        return synth.q6k_matrix_torch(gl, H, I, self.device)

    def step(self, stream=None):
        self.model.decode_step(self.X, self.M, self.ars, self.n_agents, self.rows_per_agent, self.lens,
                               self.H_out, self.ws, stream)

    def graph(self, stream):
        return self.model.graph(self.X, self.M, self.ars, self.n_agents, self.rows_per_agent, self.lens,
                                self.H_out, self.ws, stream)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during the timed region:
    NVML every 2 ms from a background thread (nvidia-smi every 100 ms if NVML is
    unavailable), so even a sub-second timed region holds many samples."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown"}

    def __init__(self, index: int):
        self.index, self.rows, self.proc, self.nv, self.stop = index, [], None, None, False
        self.source = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_sm = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.t = threading.Thread(target=self._poll_nvml, daemon=True)
            self.t.start()
            self.source = "nvml 2 ms"
            return self
        except Exception:
            self.nv = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            self.source = "nvidia-smi 100 ms"
        except FileNotFoundError:
            self.proc = None
        return self

    def _poll_nvml(self):
        nv, h = self.nv, self.h
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self.stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = get_reasons(h)
            except Exception:
                break
            reasons = [name for bit, name in self.REASONS.items() if bits & bit]
            self.rows.append((time.perf_counter(), ("nvml", sm, self.max_sm, reasons)))
            time.sleep(0.002)

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.perf_counter(), [x.strip() for x in line.split(",")]))

    def __exit__(self, *a):
        self.stop = True
        if self.nv is not None:
            self.t.join(timeout=1)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        """Samples taken between host times t0 and t1 (the timed region)."""
        rows = [r for t, r in self.rows if (t0 is None or t >= t0) and (t1 is None or t <= t1)]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        if rows[0][0] == "nvml":
            sm = [float(r[1]) for r in rows]
            mx = [float(r[2]) for r in rows]
            reasons = sorted({x for r in rows for x in r[3]})
        else:
            sm = [float(r[1]) for r in rows if len(r) > 2 and r[1].replace(".", "").isdigit()]
            mx = [float(r[2]) for r in rows if len(r) > 2 and r[2].replace(".", "").isdigit()]
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            reasons = sorted({names[i] for r in rows for i in range(4)
                              if len(r) > 5 + i and r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "source": self.source}


# ------------------------------------------------------------------ helpers

def measured_bf16_tflops(sustained=False):
    """Dense bf16 tensor throughput from MEASURED_PEAKS.json (fp16 runs at the same rate)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        v = d.get("bf16_tflops_sustained" if sustained else "bf16_tflops")
        if v:
            return float(v)
    return 1590.0


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), "measured"
    return 6650.0, "fallback"


def kernel_traffic(kernel_file: str, record: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current source of the kernel (else None)."""
    p = os.path.join(ROOT, "profiles", record)
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    src = os.path.join(ROOT, "quantized_agent_decode_b200", "csrc", kernel_file)
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return d.get("dram_bytes_per_launch") if d.get("source_sha") == h else None


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def max_over_ranks(x: float, ws: int) -> float:
    """The slowest rank's time: every rank calls this with its own measurement."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weight_stream_gbs(weight_bytes_per_gpu: int, n_gpus: int, ms_per_step: float) -> float:
    """Whole-job weight-stream rate: every replica streams its own copy of the
    weights once per step, in the slowest rank's step time."""
    return weight_bytes_per_gpu * n_gpus / (ms_per_step / 1e3) / 1e9


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle (baseline and reference arm)

_SAMPLE_CACHE = {}


def oracle_layer_sample(seed=SEED, ctx=1024, rows_per_agent=3, n_agents=4, threads=0, kv_q8=False):
    """One decoder layer of the same stack through the fp64 CPU oracle (inputs
    drawn once and reused). Returns (seconds, weight bytes of the layer, threads used)."""
    import oracle
    key = (seed, ctx, rows_per_agent, n_agents, kv_q8)
    if key not in _SAMPLE_CACHE:
        _SAMPLE_CACHE[key] = _oracle_layer_inputs(seed, ctx, rows_per_agent, n_agents, kv_q8)
    Wqkv, Wo, Wgu, Wd, Kc0, Vc0, h0, ars, lens, cap = _SAMPLE_CACHE[key]
    sh = synth.StackShape(n_layers=1)
    cp = lambda c: tuple(a.copy() for a in c) if isinstance(c, tuple) else c.copy()  # noqa: E731
    Kc, Vc, h = cp(Kc0), cp(Vc0), h0.copy()
    nth = threads or oracle.max_threads()
    t0 = time.perf_counter()
    oracle.decode_layer(Wqkv, Wo, Wgu, Wd, sh.hidden, sh.inter, sh.n_qh, sh.n_kvh, sh.head_dim, h, ars, lens,
                        Kc, Vc, cap, nthreads=nth)
    dt = time.perf_counter() - t0
    wbytes = Wqkv.size + Wo.size + Wgu.size + Wd.size
    return dt, wbytes, nth


def _oracle_layer_inputs(seed, ctx, rows_per_agent, n_agents, kv_q8=False):
    import oracle
    sh = synth.StackShape(n_layers=1)
    H, I, hd = sh.hidden, sh.inter, sh.head_dim
    nq, nkv = sh.n_qh * hd, sh.n_kvh * hd
    Wqkv = np.concatenate([synth.q4k_matrix_np(seed, 1, nq, H), synth.q4k_matrix_np(seed, 2, nkv, H),
                           synth.q4k_matrix_np(seed, 3, nkv, H)])
    Wo = synth.q4k_matrix_np(seed, 4, H, nq)
    Wgu = np.concatenate([synth.q4k_matrix_np(seed, 5, I, H), synth.q4k_matrix_np(seed, 6, I, H)])
    Wd = synth.q6k_matrix_np(seed, 7, H, I)
    cap = ctx + rows_per_agent
    if kv_q8:
        g = synth.torch_gen(seed, "cpu", 8)
        planes = []
        for _ in range(2):
            c8, s16 = synth.q8_planes_torch(g, n_agents * sh.n_kvh * cap, hd, "cpu")
            planes.append((c8.numpy().reshape(n_agents, sh.n_kvh, cap, hd),
                           s16.numpy().view(np.uint16).reshape(n_agents, sh.n_kvh, cap, hd // 32)))
        Kc, Vc = planes
    else:
        Kc = synth.bf16_normal_np(seed, 8, (n_agents, sh.n_kvh, cap, hd))
        Vc = synth.bf16_normal_np(seed, 9, (n_agents, sh.n_kvh, cap, hd))
    M = rows_per_agent * n_agents
    h = oracle.bf16_array_to_f64(synth.bf16_normal_np(seed, 10, (M, H)))
    ars = np.arange(0, M + 1, rows_per_agent, dtype=np.int32)
    lens = np.full(n_agents, ctx, np.int32)
    return Wqkv, Wo, Wgu, Wd, Kc, Vc, h, ars, lens, cap


def run_reference(args, ws, rank):
    """The oracle, as it stands, on the host cores: each step one decoder layer of
    the workload (1/64 of a decode step), extrapolated to the full step."""
    if rank != 0:
        return 0
    desc, L, rpa, na, cl = WORKLOADS[args.workload]
    for _ in range(args.warmup):
        oracle_layer_sample(ctx=cl, rows_per_agent=rpa, n_agents=na, kv_q8=args.workload in KV_Q8_WORKLOADS)
    times = []
    for _ in range(args.steps):
        dt, wb, nth = oracle_layer_sample(ctx=cl, rows_per_agent=rpa, n_agents=na,
                                          kv_q8=args.workload in KV_Q8_WORKLOADS)
        times.append(dt)
    t = statistics.median(times)
    step_s = t * L
    val = wb * L / step_s / 1e9
    line = {"metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
            "config": {"workload": desc, "rows": rpa * na, "layers": L, "cached_tokens": cl,
                       "parallelism": f"replicas{args.gpus}"},
            "cpu_baseline": {"value": val, "unit": "GB/s", "cores": nth, "kind": "oracle",
                             "sample": f"one decoder layer per step (1/{L} of a decode step), median of "
                                       f"{args.steps}, extrapolated x{L}"},
            "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

def time_gate_up(w, stream, reps=5):
    """Device time per gate|up call (prep + Q4_K GEMM) over the stack's 64 matrices:
    the calls are captured once as a graph and replayed; returns (us per call,
    algorithmic bytes per call: weights + bf16 input rows + fp32 output rows)."""
    import quantized_agent_decode_b200 as q
    sh = w.shape
    N, K, M = 2 * sh.inter, sh.hidden, w.M
    X = synth.bf16_normal_torch(synth.torch_gen(w.seed, "cuda", 4242), (M, K), "cuda")
    Y = torch.zeros(M, N, device="cuda")
    ws = q.alloc_ws(q.gemm_ws_bytes(K, M))
    with torch.cuda.stream(stream):
        for W in w.w_gu:
            q.q4k_gemm(W, N, K, X, M, Y, ws=ws, stream=stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for W in w.w_gu:
                q.q4k_gemm(W, N, K, X, M, Y, ws=ws, stream=stream)
        graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    stream.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * len(w.w_gu))
    nbytes = w.w_gu[0].numel() + M * K * 2 + M * N * 4
    del graph
    return us, nbytes


def run_gpu(args, ws, rank, local):
    import quantized_agent_decode_b200 as q
    from quantized_agent_decode_b200 import build
    if rank == 0 or not os.path.exists(q.LIB_PATH):
        build.build()
    barrier(ws)
    w = Workload(args.workload)
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()

    # graph-replayed timed region
    g = w.graph(stream)
    for _ in range(args.warmup):
        g.launch(stream)
    stream.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        t_beg = time.perf_counter()
        e0.record(stream)
        for _ in range(args.steps):
            g.launch(stream)
        e1.record(stream)
        stream.synchronize()
        t_end = time.perf_counter()
        time.sleep(0.2)
    barrier(ws)
    torch.cuda.synchronize()
    ms_step = max_over_ranks(e0.elapsed_time(e1) / args.steps, ws)
    status = q.device_status(reset=True)

    # end to end through the public API: each step packs the agents' rows on the host
    # (qad_pack_rows), copies them from pinned host memory, runs the step
    # (qad_decode_step_host: H2D, graph replay, D2H of the final hidden rows) and
    # waits for the result
    agent_rows = [w.X[a * w.rows_per_agent:(a + 1) * w.rows_per_agent].cpu() for a in range(w.n_agents)]
    lens_list = w.lens.cpu().tolist()
    Xh = torch.empty(w.M, w.shape.hidden, dtype=torch.bfloat16).pin_memory()
    arsh = torch.empty(w.n_agents + 1, dtype=torch.int32).pin_memory()
    lensh = w.lens.cpu().pin_memory()
    Hh = torch.empty(w.M, w.shape.hidden, dtype=torch.float32).pin_memory()

    def e2e_step():
        Xp, _, _, ars_p = q.pack_rows(agent_rows, lens_list, w.shape.hidden)
        Xh.copy_(Xp)
        arsh.copy_(ars_p)
        w.model.decode_step_host(Xh, w.M, arsh, w.n_agents, w.rows_per_agent, lensh, Hh, w.ws, stream)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    barrier(ws)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        e2e_step()
    e2e_ms = max_over_ranks((time.perf_counter() - t0) * 1e3 / args.steps, ws)
    h2d = Xh.numel() * 2 + arsh.numel() * 4 + lensh.numel() * 4
    d2h = Hh.numel() * 4
    g.close()

    # dominant kernel: the gate|up Q4_K GEMM (largest matrix of the layer), timed
    # over all 64 layers' matrices (6.4 GB, far above L2) as one replayed graph
    gu_us, gu_bytes = time_gate_up(w, stream)
    if rank != 0:
        return 0
    peak, peak_kind = measured_peaks()
    L = w.shape.n_layers
    achieved = gu_bytes / (gu_us * 1e-6) / 1e9
    value = weight_stream_gbs(w.weight_bytes, ws, ms_step)
    cpu = {}
    if ws == 1 and not args.no_cpu_baseline:
        # repeat one decoder layer of the same stack (fresh caches each time) for >= 10 s of CPU work
        tot, n = 0.0, 0
        while tot < 10.0 and n < L:
            dt, wb, nth = oracle_layer_sample(ctx=w.ctx, rows_per_agent=w.rows_per_agent, n_agents=w.n_agents,
                                              kv_q8=w.kv_q8)
            tot += dt
            n += 1
        cpu = {"value": wb * n / tot / 1e9, "unit": "GB/s", "cores": nth, "kind": "oracle",
               "sample": f"{n} passes of one decoder layer of the same stack ({n}/{L} of a decode step), fp64, "
                         f"{tot:.1f} s; the full step extrapolates to {tot / n * L * 1e3:.0f} ms"}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16xf16->f32 (tensor-core operands exact), bf16 KV/activations",
        "data": "synthetic (seeded, drawn in device memory)",
        "config": {"workload": w.desc, "rows": w.M, "agents": w.n_agents, "layers": L,
                   "cached_tokens": w.ctx, "weight_bytes_per_step": w.weight_bytes,
                   "kv_bytes_per_step": w.kv_bytes, "parallelism": f"replicas{ws}",
                   "l2": "inputs larger than L2 (13.7 GB of weights per step), no flush"},
        "roofline": {"bound": "hbm", "kernel": "q4k gate|up GEMM (N=34816, K=5120, M=12)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": peak_kind,
                     "traffic": kernel_traffic("gemm.cu", "q4k_gemm_gate_up_traffic.json"),
                     "duration_us": gu_us, "bytes_per_launch": gu_bytes,
                     "timing": "CUDA events on the replaying stream around a graph of the 64 layers' gate|up "
                               "calls (prep + GEMM each; the time includes the prep)"},
        "step_stream_gbs": (w.weight_bytes + w.kv_bytes) / (ms_step / 1e3) / 1e9,
        "kernel_shares": "profiles/step_launches_stack12_ctx1k.md (ncu launch list)",
        "e2e": {"value": weight_stream_gbs(w.weight_bytes, ws, e2e_ms), "unit": "GB/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": w.model.launches() * args.steps,
        "clocks": clk.summary(t_beg, t_end),
        "device_status": status,
    }
    if cpu:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)
    return 0


DENSE_KERNELS = {  # prefill chunk (2048 prompt rows + 12 decode rows) through one matrix: (format, N, K, M)
    "pf_gate_up": (4, 34816, 5120, 2060), "pf_down": (6, 5120, 17408, 2060), "pf_qkv": (4, 8192, 5120, 2060),
    "pf_o": (4, 5120, 6144, 2060),
}

STEP_LAUNCHES = ["prep_rms_attn", "gemm_qkv", "attn", "prep_merge", "gemm_o", "prep_rms_mlp", "gemm_gate_up",
                 "prep_silu", "gemm_down"]


def run_trace(args):
    """Per-launch device timeline of one replayed step (qad_model_set_trace): for each
    launch kind the mean wait (start -> dependency met), run (-> last warp exit) and
    critical-path share (previous launch's end -> this launch's end), in microseconds."""
    from quantized_agent_decode_b200 import build
    build.build()
    w = Workload(args.workload)
    stream = torch.cuda.Stream()
    w.model.set_trace(True)
    g = w.graph(stream)
    for _ in range(max(args.warmup, 1)):
        g.launch(stream)
    stream.synchronize()
    w.model.trace_reset()
    torch.cuda.synchronize()
    g.launch(stream)
    stream.synchronize()
    t = w.model.trace_read().numpy() / 1000.0
    names = ["init"] + STEP_LAUNCHES * w.shape.n_layers
    kinds, prev = {}, 0.0
    for i, nm in enumerate(names):
        st, rd, en = t[i]
        d = kinds.setdefault(nm, [0, 0.0, 0.0, 0.0])
        d[0] += 1
        d[1] += rd - st
        d[2] += en - rd
        d[3] += en - prev
        prev = en
    out = {"workload": w.desc, "step_us": round(float(t[:, 2].max()), 1),
           "per_launch_kind_us": {k: {"wait": round(v[1] / v[0], 2), "run": round(v[2] / v[0], 2),
                                      "critical": round(v[3] / v[0], 2), "per_step": v[0]} for k, v in kinds.items()}}
    print(json.dumps(out), flush=True)
    g.close()
    return 0


KERNELS = {  # single-kernel cases for profiler captures: (format, N, K)
    "qkv": (4, 8192, 5120), "o": (4, 5120, 6144), "gate_up": (4, 34816, 5120), "down": (6, 5120, 17408),
    "gate": (4, 17408, 5120),  # one MLP gate (or up) projection alone
}


def run_kernel(args):
    """Time one matrix of the stack through the public GEMM entry point (prep +
    GEMM per call), rotating 8 weight copies so every call streams from HBM; the
    8 calls are replayed as one CUDA graph, so the time is device time."""
    import quantized_agent_decode_b200 as q
    from quantized_agent_decode_b200 import build
    build.build()
    g = synth.torch_gen(SEED, "cuda", 77)
    if args.kernel in DENSE_KERNELS:
        fmt, N, K, M = DENSE_KERNELS[args.kernel]
        mk = synth.q4k_matrix_torch if fmt == 4 else synth.q6k_matrix_torch
        Ws = [mk(g, N, K, "cuda") for _ in range(2)]
        if fmt == 6:
            Ws = [q.q6k_pack(w, N, K) for w in Ws]
        X = synth.bf16_normal_torch(g, (M, K), "cuda")
        Y = torch.empty(M, N, device="cuda")
        ws = q.alloc_ws(q.dense_gemm_ws_bytes(K, M))
        gemm = q.q4k_gemm_dense if fmt == 4 else q.q6k_gemm_dense
        fn = lambda i, st: gemm(Ws[i % 2], N, K, X, M, Y, ws=ws, stream=st)  # noqa: E731
        nbytes = Ws[0].numel()
        flops = 2.0 * M * N * K
    elif args.kernel == "verify":
        hidden, vocab, M = 5120, 151936, 12
        Wh = synth.q4k_matrix_torch(g, vocab, hidden, "cuda")
        Hd = synth.bf16_normal_torch(g, (M, hidden), "cuda").float()
        ars = torch.arange(0, 13, 3, dtype=torch.int32, device="cuda")
        toks = torch.randint(0, vocab, (M,), generator=g, dtype=torch.int32, device="cuda")
        lens = torch.full((4,), 1024, dtype=torch.int32, device="cuda")
        out = torch.empty(M, dtype=torch.int32, device="cuda")
        acc = torch.empty(4, dtype=torch.int32, device="cuda")
        ws = q.alloc_ws(q.verify_ws_bytes(hidden, vocab, M))
        fn = lambda i, st: q.verify_step(Hd, M, hidden, Wh, vocab, ars, 4, toks, lens, out, acc, ws=ws,  # noqa: E731
                                         stream=st)
        nbytes = Wh.numel()
    elif args.kernel == "pfattn23k":
        len_, C, n_qh, n_kvh = 23000, 2048, 48, 8
        cap = len_ + C
        Kd = synth.bf16_normal_torch(g, (n_kvh, cap, 128), "cuda")
        Vd = synth.bf16_normal_torch(g, (n_kvh, cap, 128), "cuda")
        Qd = synth.bf16_normal_torch(g, (C, n_qh, 128), "cuda")
        O = torch.zeros(C, n_qh, 128, dtype=torch.bfloat16, device="cuda")
        fn = lambda i, st: q.prefill_attn(Qd, Kd, Vd, len_, C, cap, n_qh, n_kvh, 128, O, stream=st)  # noqa: E731
        nbytes = 2 * n_kvh * cap * 128 * 2
        # QK^T and PV over the visible keys: row j sees len + j + 1 keys
        flops = 4.0 * 128 * n_qh * (C * (len_ + 1) + C * (C - 1) / 2)
    elif args.kernel == "attn23k":
        A, L, n_qh, n_kvh = 4, 23000, 48, 8
        cap = L + 3
        Kd = synth.bf16_normal_torch(g, (A, n_kvh, cap, 128), "cuda")
        Vd = synth.bf16_normal_torch(g, (A, n_kvh, cap, 128), "cuda")
        Qd = synth.bf16_normal_torch(g, (12, n_qh, 128), "cuda")
        lens = torch.full((A,), L, dtype=torch.int32, device="cuda")
        ars = torch.arange(0, 13, 3, dtype=torch.int32, device="cuda")
        O = torch.zeros(12, n_qh, 128, dtype=torch.bfloat16, device="cuda")
        ws = q.alloc_ws(q.decode_attn_ws_bytes(A, n_qh, n_kvh, cap, 3))
        fn = lambda i, st: q.decode_attn(Qd, Kd, Vd, lens, ars, A, 3, cap, n_qh, n_kvh, 128, O, ws=ws,  # noqa: E731
                                         stream=st)
        nbytes = 2 * A * n_kvh * cap * 128 * 2
    elif args.kernel == "attn23k_q8":
        A, L, n_qh, n_kvh = 4, 23000, 48, 8
        cap = L + 3
        Kq, Kd = synth.q8_planes_torch(g, A * n_kvh * cap, 128, "cuda")
        Vq, Vd = synth.q8_planes_torch(g, A * n_kvh * cap, 128, "cuda")
        Kd, Vd = Kd.view(torch.int16), Vd.view(torch.int16)
        Qd = synth.bf16_normal_torch(g, (12, n_qh, 128), "cuda")
        lens = torch.full((A,), L, dtype=torch.int32, device="cuda")
        ars = torch.arange(0, 13, 3, dtype=torch.int32, device="cuda")
        O = torch.zeros(12, n_qh, 128, dtype=torch.bfloat16, device="cuda")
        ws = q.alloc_ws(q.decode_attn_ws_bytes(A, n_qh, n_kvh, cap, 3))
        fn = lambda i, st: q.decode_attn_q8(Qd, Kq, Kd, Vq, Vd, lens, ars, A, 3, cap, n_qh, n_kvh, 128,  # noqa: E731
                                            O, ws=ws, stream=st)
        nbytes = 2 * A * n_kvh * cap * (128 + 8)
    else:
        fmt, N, K = KERNELS[args.kernel]
        mk = synth.q4k_matrix_torch if fmt == 4 else synth.q6k_matrix_torch
        Ws = [mk(g, N, K, "cuda") for _ in range(8)]
        if fmt == 6:
            Ws = [q.q6k_pack(w, N, K) for w in Ws]
        M = args.rows
        X = synth.bf16_normal_torch(g, (M, K), "cuda")
        Y = torch.zeros(M, N, device="cuda")
        ws = q.alloc_ws(q.gemm_ws_bytes(K, M))
        gemm = q.q4k_gemm if fmt == 4 else q.q6k_gemm
        fn = lambda i, st: gemm(Ws[i % 8], N, K, X, M, Y, ws=ws, stream=st)  # noqa: E731
        nbytes = Ws[0].numel()
    if args.kernel not in DENSE_KERNELS and args.kernel != "pfattn23k":
        flops = None
    # 8 calls (8 weight copies) captured once and replayed: device time only, no host launch cost
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for i in range(8):
            fn(i, stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(8):
            fn(i, stream)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(1, args.steps // 8)
    e0.record()  # graph.replay() launches on the current stream
    for _ in range(reps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) / (reps * 8) * 1e3
    out = {"kernel": args.kernel, "rows": args.rows, "us_per_call": us, "gbs": nbytes / us / 1e3, "bytes": nbytes,
           "device_status": q.device_status()}
    if flops:
        peak = measured_bf16_tflops()
        out.update({"rows": DENSE_KERNELS[args.kernel][3] if args.kernel in DENSE_KERNELS else 2048,
                    "tflops": flops / us / 1e6, "flop_per_call": flops,
                    "peak_tflops": peak, "frac": flops / us / 1e6 / peak if peak else None,
                    "dense_status": q.dense_status() if args.kernel in DENSE_KERNELS else None})
    print(json.dumps(out), flush=True)
    return 0


def run_sched(args):
    """Decode rate of three agents (1024 cached tokens, 12-row budget) while a
    fourth agent's 20480-token prompt is fed through the 64-layer stack in
    2048-row chunks, under three scheduler policies (host planner of the
    library; decode steps and mixed decode+chunk steps timed with CUDA events).
    The synthetic weights accept no drafts, so each decoding agent gains one
    token per step it is scheduled in."""
    import quantized_agent_decode_b200 as q
    from quantized_agent_decode_b200 import build
    build.build()
    PROMPT, CTX, CHUNK, A = 20480, 1024, 2048, 4
    w = Workload("stack12_ctx1k", ctx=PROMPT + 16)
    H = w.shape.hidden
    g = synth.torch_gen(SEED, "cuda", 91)
    X = synth.bf16_normal_torch(g, (12 + CHUNK, H), "cuda")
    Hout = torch.empty(12 + CHUNK, H, dtype=torch.float32, device="cuda")
    ws_mix = q.alloc_ws(w.model.mixed_ws_bytes(12, CHUNK))
    ars_d = torch.zeros(A + 1, dtype=torch.int32, device="cuda")
    lens_d = torch.zeros(A, dtype=torch.int32, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def run_step(rows, ca, cr, lens):
        M = sum(rows)
        ars = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
        ars_d.copy_(torch.from_numpy(ars))
        lens_d.copy_(torch.from_numpy(np.array(lens, np.int32)))
        e0.record()
        if cr:
            w.model.mixed_step(X[:M + cr], M, ars_d if M else None, A, max(max(rows), 1), lens_d if M else None,
                               ca, lens[ca], cr, Hout, ws_mix)
        else:
            w.model.decode_step(X[:M], M, ars_d, A, max(rows), lens_d, Hout, w.ws)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    # warm-up: one decode step and one mixed step (the chunk rows land in the prompt agent's cache, later overwritten)
    run_step([3, 3, 3, 0], -1, 0, [CTX, CTX, CTX, 0])
    run_step([3, 3, 3, 0], 3, CHUNK, [CTX, CTX, CTX, 0])
    decode_ms = statistics.median(run_step([3, 3, 3, 0], -1, 0, [CTX, CTX, CTX, 0]) for _ in range(10))
    out = {"workload": "64-layer stack; agents 0-2 decoding at 1024 cached tokens (1 token + 2 drafts each), "
                       "agent 3 with a 20480-token prompt fed in 2048-row chunks",
           "decode_step_ms": round(decode_ms, 3), "decode_tok_s_per_agent_alone": round(1e3 / decode_ms, 1),
           "policies": {}}
    for name, mode, every in (("interleave_every_step", q.SCHED_INTERLEAVE, 0),
                              ("interleave_every_4th_step", q.SCHED_INTERLEAVE, 3),
                              ("prefill_first", q.SCHED_PREFILL_FIRST, 0)):
        s = q.Scheduler(A, chunk_tokens=CHUNK, decode_steps_per_chunk=every, max_decode_rows=12, n_draft=2, mode=mode)
        for a in range(A):
            s.agents[a].len, s.agents[a].prompt_left, s.agents[a].active, s.agents[a].drafts = CTX, 0, 1, 2
        s.agents[3].len, s.agents[3].prompt_left = 0, PROMPT
        total, dec, chunk_ms, steps = 0.0, 0, [], 0
        while s.agents[3].prompt_left > 0:
            rows, ca, cr = s.plan()
            ms = run_step(rows, ca, cr, [s.agents[a].len for a in range(A)])
            total += ms
            if cr:
                chunk_ms.append(round(ms, 1))
            dec += rows[0] > 0
            s.commit(rows, ca, cr, n_accept=[0] * A)
            for a in range(3):
                s.agents[a].drafts = 2
            steps += 1
        out["policies"][name] = {"time_to_prompt_ms": round(total, 1), "steps": steps,
                                 "decode_tokens_per_agent": dec,
                                 "decode_tok_s_per_agent_during_prompt": round(dec / total * 1e3, 1),
                                 "chunk_step_ms": chunk_ms}
    out["device_status"] = q.device_status()
    out["dense_status"] = q.dense_status()
    print(json.dumps(out), flush=True)
    return 0


def run_ttft(args):
    """Next-request time to first token with and without KV reuse: agents 0-2 keep
    decoding (1024 cached tokens, 1 token + 2 drafts each) while agent 3, whose
    cache holds its previous 23000-token context, sends a request that appends 512
    new tokens. With reuse (qad_common_prefix of the old and new token sequences)
    only the suffix is prefilled; without it the whole 23512-token prompt is fed
    from an empty cache in 2048-row chunks. Each chunk rides with the decode rows
    in one mixed step; the first token is the argmax of the vocabulary head over
    the prompt's last row. Device time by CUDA events around the whole sequence."""
    import quantized_agent_decode_b200 as q
    from quantized_agent_decode_b200 import build
    build.build()
    PREV, NEW, CHUNK, A, VOCAB = 23000, 512, 2048, 4, 151936
    w = Workload("stack12_ctx1k", ctx=PREV + NEW + 16)
    H = w.shape.hidden
    g = synth.torch_gen(SEED, "cuda", 93)
    X = synth.bf16_normal_torch(g, (9 + CHUNK, H), "cuda")
    W_head = synth.q4k_matrix_torch(g, VOCAB, H, "cuda")
    Hout = torch.empty(9 + CHUNK, H, dtype=torch.float32, device="cuda")
    ws_mix = q.alloc_ws(w.model.mixed_ws_bytes(9, CHUNK))
    ars_d = torch.tensor([0, 3, 6, 9, 9], dtype=torch.int32, device="cuda")
    lens_d = torch.zeros(A, dtype=torch.int32, device="cuda")
    head_ars = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    head_tok = torch.zeros(1, dtype=torch.int32, device="cuda")
    head_len = torch.zeros(1, dtype=torch.int32, device="cuda")
    first_tok = torch.zeros(1, dtype=torch.int32, device="cuda")
    n_acc = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws_head = q.alloc_ws(q.verify_ws_bytes(H, VOCAB, 1))
    rng = np.random.default_rng(SEED)
    old_tokens = rng.integers(0, VOCAB, PREV).tolist()
    new_tokens = old_tokens + rng.integers(0, VOCAB, NEW).tolist()

    def request(start):
        """Prefill new_tokens[start:] of agent 3 in chunks beside the decode rows, then the head."""
        pos = start
        while pos < len(new_tokens):
            C = min(CHUNK, len(new_tokens) - pos)
            lens_d.copy_(torch.tensor([1024, 1024, 1024, pos], dtype=torch.int32))
            w.model.mixed_step(X[:9 + C], 9, ars_d, A, 3, lens_d, 3, pos, C, Hout, ws_mix)
            pos += C
        q.verify_step(Hout[8 + C:9 + C], 1, H, W_head, VOCAB, head_ars, 1, head_tok, head_len, first_tok, n_acc,
                      ws=ws_head)
        return pos

    def timed(start):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        request(start)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    reuse = q.common_prefix(old_tokens, new_tokens)
    timed(reuse)  # warm-up of both shapes
    timed(PREV + NEW - CHUNK)
    t_reuse = statistics.median(timed(reuse) for _ in range(5))
    t_full = statistics.median(timed(0) for _ in range(2))
    out = {"workload": "64-layer stack; agents 0-2 decoding at 1024 cached tokens (3 rows each) while agent 3 "
                       f"sends a request of {NEW} new tokens after a {PREV}-token context",
           "reused_prefix_tokens": reuse, "chunk_rows": CHUNK,
           "ttft_ms_with_kv_reuse": round(t_reuse, 2),
           "ttft_ms_without_reuse": round(t_full, 2),
           "speedup": round(t_full / t_reuse, 1),
           "mixed_steps": {"with_reuse": -(-NEW // CHUNK), "without": -(-(PREV + NEW) // CHUNK)},
           "head": f"Q4_K vocabulary head {VOCAB} x {H}, argmax of the prompt's last row",
           "device_status": q.device_status(), "dense_status": q.dense_status()}
    print(json.dumps(out), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)  # ~2.4 s timed at ~6 ms per step
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="stack12_ctx1k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=sorted(list(KERNELS) + list(DENSE_KERNELS) + ["attn23k", "attn23k_q8", "pfattn23k", "verify"]),
                    help="time one kernel of the step instead (profiler captures)")
    ap.add_argument("--rows", type=int, default=12)
    ap.add_argument("--trace", action="store_true", help="print the per-launch device timeline of one step")
    ap.add_argument("--ttft", action="store_true",
                    help="next-request time to first token with and without KV reuse (23000-token context)")
    ap.add_argument("--sched", action="store_true",
                    help="decode rate of three agents while a 20480-token prompt is chunked in (scheduler policies)")
    args = ap.parse_args()
    if args.sched:
        return run_sched(args)
    if args.ttft:
        return run_ttft(args)
    if args.kernel:
        return run_kernel(args)
    if args.trace:
        return run_trace(args)
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: re-launch under torch.distributed.run on this node
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
        return subprocess.call(cmd)
    ws, rank, local = (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                       int(os.environ.get("LOCAL_RANK", "0")))
    if ws != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={ws}", file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args, ws, rank)
    ws, rank, local = dist_setup()
    try:
        return run_gpu(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
