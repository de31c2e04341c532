"""Benchmark of the hybrid-precision attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one layer, Llama-3.1-8B attention shape at a 32K prefix): B=1,
Hq=32, Hkv=8, D=128, prefix L=32768, rho=5 %, W=128, K4V4 groups of 32, the
planted-vertical-line generator of ``hybrid_precision_attention_b200.synth``.

One bench step = one 64-token reselection period: 64 decode tokens, then a
vertical-line reselection and a staging -> hybrid merge.  The layer is held as
8 independent copies that are visited in turn (token t runs copy 0..7), so
the working set (~400 MB) is larger than the 126 MB L2 and every decode reads
its cache from HBM; per step that is 512 decode launches plus 8 selections
and 8 merges, replayed from two CUDA graphs with CUDA events between the
replays.  The reported metric is the decode-attention throughput of the whole
period: algorithmic bytes of the 512 decode steps divided by the time of the
whole step (decode + selection + merge), in GB/s, with microseconds per
decode token-layer alongside.

Algorithmic bytes of one decode step of one (b, kv head): 160 B per K4V4
position outside the vertical-line set (64 + 16 bytes of K codes/scales and the
same for V), 512 B per FP16 position (vertical lines, recent window and staged
tokens, the new token included), plus the query and output rows.  A vertical
line's key and value are read from the VL store; the K4V4 record that its page
still carries is layout overhead, seen in the ncu traffic, not counted here.

Multi-GPU: the path has no exchange step; ``--gpus N`` (under torchrun) runs N
independent replicas, one per GPU, the timing is the max over ranks and the
value the sum of all ranks' bytes over that time (weak scaling).

``--impl reference`` times the CPU oracle (``oracle/``) on the host cores on a
bounded sample of the same workload (single decode steps of the 32K layer).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn µs/step & achieved HBM GB/s (% of B200 peak) at 32K context"
UNIT = "GB/s"
B, HQ, HKV, D, L, W, RHO_BP = 1, 32, 8, 128, 32768, 128, 500
COPIES = 8
PERIOD = 64
WORKLOAD = ("decode attention over a hybrid K4V4/FP16 cache, one layer: B=1, Hq=32, Hkv=8 (GQA 4), D=128, "
            "prefix 32768, rho=5%, W=128, K4V4 group 32, planted vertical lines; step = 64 decode tokens + "
            "reselection + merge on each of 8 rotating layer copies")


def k_of(n, rho_bp):
    return 0 if n <= 0 or rho_bp <= 0 else min(n, (n * rho_bp + 9999) // 10000)


def decode_bytes(n_packed, n_vl, T):
    """Algorithmic bytes of one decode step (all kv heads) at the given state (before the step):
    packed positions outside the VL set at 160 B, FP16 rows (VL, ring, new token) at 512 B."""
    fp16_rows = n_vl + (T + 1 - n_packed)
    per_head = (n_packed - n_vl) * 160 + fp16_rows * 512
    return B * HKV * per_head + 2 * B * HQ * D * 2


def period_bytes(T0):
    """Algorithmic decode bytes of one 64-token period starting right after a merge at length T0."""
    n_packed = T0 - W
    n_vl = k_of(n_packed, RHO_BP)
    return sum(decode_bytes(n_packed, n_vl, T0 + t) for t in range(PERIOD))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def load_bf16_peak():
    """Dense bf16 tensor peak (TFLOP/s): the burst figure, for a kernel timed on its own."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


PF_L, PF_HQ, PF_HKV = 32768, 32, 8


def prefill_flops(L, Hq, D=128):
    """Algorithmic FLOPs of causal attention: 2 GEMMs x 2 flops x D x Hq x L(L+1)/2."""
    return 4.0 * D * Hq * L * (L + 1) / 2


def run_prefill(dev, reps=5, warmup=2):
    """Time hq_prefill_attn on the 32K layer (B=1, Hq=32, Hkv=8, W=128, 5 % vertical lines chosen
    from the column mass of the last 64 queries); returns the JSON object of the prefill leg."""
    import torch
    from hybrid_precision_attention_b200 import hq, synth
    lay = synth.planted_layer(0, 1, PF_HQ, PF_HKV, PF_L)
    Q = synth.full_queries(0, 1, PF_HQ, PF_HKV, PF_L)
    q_d = torch.from_numpy(Q).to(dev)
    k_d, v_d = torch.from_numpy(lay.k).to(dev), torch.from_numpy(lay.v).to(dev)
    # vertical lines from the prompt's own last 64 queries
    c = hq.HybridCache(1, PF_HQ, PF_HKV, PF_L, W, RHO_BP, device=dev)
    hq.hq_select_vlines(c, k_d, q_d[:, :, PF_L - 64:].contiguous())
    torch.cuda.synchronize()
    n_vl = c.state()["k_sel"]
    vl = c.vl_sel
    out = torch.empty_like(q_d)
    ws = torch.empty(hq.hq_prefill_workspace_bytes(1, PF_HQ, PF_HKV, PF_L), dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        hq.hq_prefill_attn(q_d, k_d, v_d, vl, n_vl, W, out=out, ws=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        hq.hq_prefill_attn(q_d, k_d, v_d, vl, n_vl, W, out=out, ws=ws)
    e1.record()
    torch.cuda.synchronize()
    err = int(ws[:4].cpu().numpy().view(np.uint32)[0])
    assert err == 0, err
    ms = e0.elapsed_time(e1) / reps
    flops = prefill_flops(PF_L, PF_HQ)
    tflops = flops / (ms * 1e-3) / 1e12
    bf16, kind = load_bf16_peak()
    fp8 = 2.0 * bf16
    mixed = 1.0 / (0.5 / fp8 + 0.5 / bf16)
    return {"workload": f"causal hybrid prefill, B=1, L=32768, Hq=32, Hkv=8, D=128, W=128, rho=5% ({n_vl} lines per kv head)",
            "ms": ms, "tflops": tflops, "calls": reps,
            "roofline": {"kernel": "prefill (pre-pass + prefill_kernel)", "bound": "tensor", "achieved": tflops,
                         "peak": fp8, "unit": "TFLOP/s", "frac": tflops / fp8, "traffic": None,
                         "peak_kind": f"{kind} bf16 x 2 (nominal fp8/bf16 ratio)",
                         "mixed_ceiling": mixed,
                         "note": "QK of quantised tiles on e4m3 (fp8 rate), P.V on f16 (bf16 rate): half the flops at "
                                 "each rate, so the ceiling of this mix is the mixed_ceiling figure"}}


def decode_traffic_record():
    """DRAM bytes per decode launch from the committed ncu summary, if it matches the current kernel source."""
    src = open(os.path.join(ROOT, "hybrid_precision_attention_b200", "csrc", "decode.cu"), "rb").read()
    sha = hashlib.sha256(src).hexdigest()
    p = os.path.join(ROOT, "profiles", "decode_kernel_32k.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m_sha = re.search(r"decode\.cu sha256:\s*([0-9a-f]{64})", txt)
    m_b = re.search(r"dram bytes per launch \(read \+ write\):\s*([0-9]+)", txt)
    if not m_sha or not m_b or m_sha.group(1) != sha:
        return None
    return int(m_b.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every INTERVAL_MS from
    start() on (nvidia-smi needs a moment before its first sample, so start it
    before the warm-up); summary() keeps the samples whose own timestamps fall
    between begin() and end(), i.e. inside the timed region."""

    INTERVAL_MS = 25
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        # nvidia-smi numbers GPUs physically; under CUDA_VISIBLE_DEVICES the
        # process's device `index` is the index-th entry of that list (an index
        # or a UUID, both of which nvidia-smi -i accepts)
        visible = [x.strip() for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
        self.index = visible[index] if index < len(visible) else str(index)
        self.proc = None
        self.lines = []
        self.t_begin = self.t_end = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def begin(self):
        self.t_begin = datetime.datetime.now()

    def end(self):
        self.t_end = datetime.datetime.now()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.t.join(timeout=5)

    def __enter__(self):
        self.start()
        self.begin()
        return self

    def __exit__(self, *a):
        self.end()
        self.stop()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        slack = datetime.timedelta(milliseconds=self.INTERVAL_MS)
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
            except ValueError:
                ts = None
            if ts is not None and self.t_begin is not None and self.t_end is not None:
                if ts < self.t_begin - slack or ts > self.t_end + slack:
                    continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle legs

def oracle_sample(min_seconds=10.0, max_steps=64, steps=None):
    """Time single oracle decode steps of the 32K layer; returns (GB/s, seconds per step, steps, threads)."""
    from hybrid_precision_attention_b200 import synth
    from oracle import hybrid
    lay = synth.planted_layer(0, B, HQ, HKV, L)
    c = hybrid.HybridCacheRef(B, HQ, HKV, W, RHO_BP, L + 1024)
    c.init_from_prefix(lay.k, lay.v, lay.q_tail)
    q, k, v = synth.decode_tokens(0, B, HQ, HKV, max_steps if steps is None else steps)
    times, nbytes = [], []
    t_start = time.perf_counter()
    i = 0
    while True:
        st = (c.n_packed, len(c.vl[0][0]), c.T)
        t0 = time.perf_counter()
        c.decode(q[i], k[i], v[i])
        times.append(time.perf_counter() - t0)
        nbytes.append(decode_bytes(*st))
        i += 1
        if steps is not None and i >= steps:
            break
        if steps is None and (time.perf_counter() - t_start >= min_seconds or i >= max_steps):
            break
    gbs = sum(nbytes) / sum(times) / 1e9
    threads = int(os.environ.get("OMP_NUM_THREADS") or os.environ.get("OPENBLAS_NUM_THREADS") or len(os.sched_getaffinity(0)))
    return gbs, float(np.mean(times)), i, threads, times, nbytes


def aggregate_ranks(ms_local, units_local, world, device):
    """The job's timed duration and work over all ranks: the max of the ranks'
    device-timed durations (the job ends with its slowest rank) and the sum of
    the units (bytes) they processed.  Every rank makes the same two collectives."""
    if world == 1:
        return float(ms_local), float(units_local)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms_local)], dtype=torch.float64, device=device)
    u = torch.tensor([float(units_local)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def run_reference(args, rank, world):
    if rank != 0:
        return
    # warm-up steps, then exactly K timed steps (each: one oracle decode step of the 32K layer)
    from hybrid_precision_attention_b200 import synth  # noqa: F401
    _, _, _, threads, times, nbytes = oracle_sample(steps=args.warmup + args.steps)
    tt = times[args.warmup:]
    bb = nbytes[args.warmup:]
    value = sum(bb) / sum(tt) / 1e9
    sample = (f"{args.steps} single decode steps of the 32K layer (B=1, Hq=32, Hkv=8) by the float64 oracle after "
              f"{args.warmup} warm-up steps; prefix install (selection + pack) not timed")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.mean(tt)) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": "single decode steps, CPU"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU leg

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from hybrid_precision_attention_b200 import hq, synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    n_steps_total = args.warmup + args.steps + 2
    cap = L + PERIOD * (n_steps_total + 4) + 256

    lay = synth.planted_layer(0, B, HQ, HKV, L)
    k_d, v_d, qt_d = [torch.from_numpy(a).to(dev) for a in (lay.k, lay.v, lay.q_tail)]
    caches = []
    for _ in range(COPIES):
        c = hq.HybridCache(B, HQ, HKV, cap, W, RHO_BP, device=dev)
        hq.hq_select_vlines(c, k_d, qt_d)
        hq.hq_pack_merge(c, k_d, v_d)
        caches.append(c)
    del k_d, v_d, qt_d
    qn, kn, vn = synth.decode_tokens(1, B, HQ, HKV, PERIOD)
    q_t, k_t, v_t = [torch.from_numpy(a).to(dev) for a in (qn, kn, vn)]
    out = torch.empty((B, HQ, D), dtype=torch.float16, device=dev)
    for c in caches:
        for op in (hq.OP_SELECT, hq.OP_MERGE, hq.OP_DECODE):
            c.workspace(op)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)

    def decode_block():
        for t in range(PERIOD):
            for c in caches:
                hq.hq_decode_attn(c, q_t[t], k_t[t], v_t[t], out=out, stream=stream)

    def maint_block():
        for c in caches:
            hq.hq_select_vlines(c, stream=stream)
            hq.hq_pack_merge(c, stream=stream)

    # one eager period first (sets function attributes, checks the state machine)
    with torch.cuda.stream(stream):
        decode_block()
        maint_block()
    stream.synchronize()
    st0 = caches[0].state()
    assert st0["err"] == 0 and st0["T"] == L + PERIOD and st0["n_packed"] == L + PERIOD - W, st0

    g_dec, g_mnt = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_dec, stream=stream):
        decode_block()
    with torch.cuda.graph(g_mnt, stream=stream):
        maint_block()
    # capture does not run the work; the caches are still at T = L + 64, just merged

    # our kernels per step: one decode_kernel per token and copy; per copy a
    # reselection (sel_pass<0>, sel_pass<1>, topk_kernel) and a staging merge
    # (pack_rows_kernel, vl_gather_kernel, vl_install_kernel)
    launches_per_step = PERIOD * COPIES + COPIES * (3 + 3)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        g_dec.replay()
        if ev is not None:
            ev[1].record(stream)
        g_mnt.replay()
        if ev is not None:
            ev[2].record(stream)

    sampler = ClockSampler(local_rank).start()  # sampling from the warm-up on; summarised over the timed region
    try:
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                step()
        stream.synchronize()
        T_first = caches[0].state()["T"]
        # timed region
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        sampler.begin()
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                step(evs[i])
        torch.cuda.synchronize()
        sampler.end()
    finally:
        sampler.stop()
    if world > 1:
        dist.barrier()
    for c in caches:
        st = c.state()
        assert st["err"] == 0, st
    dec_ms = [evs[i][0].elapsed_time(evs[i][1]) for i in range(args.steps)]
    mnt_ms = [evs[i][1].elapsed_time(evs[i][2]) for i in range(args.steps)]
    total_ms = evs[0][0].elapsed_time(evs[-1][2])
    bytes_local = sum(period_bytes(T_first + PERIOD * i) for i in range(args.steps)) * COPIES
    total_ms_max, bytes_all = aggregate_ranks(total_ms, bytes_local, world, dev)
    value = bytes_all / (total_ms_max * 1e-3) / 1e9
    n_decodes = PERIOD * COPIES * args.steps
    us_per_decode = total_ms_max * 1e3 / n_decodes
    peak, peak_kind = load_peaks()

    # roofline of the dominant kernel: decode, average launch duration over the timed region
    dec_avg_us = sum(dec_ms) * 1e3 / n_decodes
    bytes_per_launch = bytes_local / n_decodes
    achieved = bytes_per_launch / (dec_avg_us * 1e-6) / 1e9
    traffic = decode_traffic_record()
    roof = {"kernel": "decode_kernel", "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
            "avg_launch_us": dec_avg_us, "algorithmic_bytes_per_launch": bytes_per_launch}

    # end-to-end leg: the public API with host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        qh = torch.from_numpy(qn).pin_memory()
        kh = torch.from_numpy(kn).pin_memory()
        vh = torch.from_numpy(vn).pin_memory()
        outh = torch.empty((PERIOD, COPIES, B, HQ, D), dtype=torch.float16).pin_memory()
        qd = torch.empty((B, HQ, D), dtype=torch.float16, device=dev)
        kd = torch.empty((B, HKV, D), dtype=torch.float16, device=dev)
        vd = torch.empty((B, HKV, D), dtype=torch.float16, device=dev)
        n_e2e = max(1, min(args.steps, 3))
        T_e = caches[0].state()["T"]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(n_e2e):
                for tt in range(PERIOD):
                    for ci, c in enumerate(caches):
                        qd.copy_(qh[tt], non_blocking=True)
                        kd.copy_(kh[tt], non_blocking=True)
                        vd.copy_(vh[tt], non_blocking=True)
                        hq.hq_decode_attn(c, qd, kd, vd, out=out, stream=stream)
                        outh[tt, ci].copy_(out, non_blocking=True)
                maint_block()
                stream.synchronize()   # the step's results are on the host
            e1.record(stream)
        torch.cuda.synchronize()
        e_ms = e0.elapsed_time(e1)
        e_ms_max, e_bytes = aggregate_ranks(e_ms, sum(period_bytes(T_e + PERIOD * i) for i in range(n_e2e)) * COPIES,
                                            world, dev)
        e2e = {"value": e_bytes / (e_ms_max * 1e-3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": PERIOD * COPIES * (qd.numel() + kd.numel() + vd.numel()) * 2,
               "d2h_bytes_per_step": PERIOD * COPIES * out.numel() * 2,
               "steps": n_e2e, "api": "hq_decode_attn / hq_select_vlines / hq_pack_merge via the Python binding, eager"}

    prefill = None
    if not args.no_prefill:
        prefill = run_prefill(dev)

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu:
        gbs, sec, n, threads, _, _ = oracle_sample(min_seconds=args.cpu_seconds)
        cpu = {"value": gbs, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{n} single decode steps of the 32K layer by the float64 oracle ({sec:.2f} s each); "
                         f"prefix install not timed"}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "us_per_decode_step": us_per_decode, "pct_of_hbm_peak": 100.0 * value / peak,
            "select_merge_share": sum(mnt_ms) / max(sum(dec_ms) + sum(mnt_ms), 1e-9),
            "config": {"workload": WORKLOAD, "B": B, "Hq": HQ, "Hkv": HKV, "D": D, "prefix": L, "W": W,
                       "rho": RHO_BP / 10000, "layer_copies": COPIES, "decode_tokens_per_step": PERIOD,
                       "l2": f"{COPIES} rotating layer copies, {COPIES * caches[0].nbytes() / 1e6:.0f} MB working set > 126 MB L2",
                       "parallelism": f"replicas x{world}"},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "prefill": prefill,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": sampler.summary()}
    print(json.dumps(line), flush=True)


def profile_decode():
    """Small case for ncu captures: one 32K layer cache, 4 decode steps with an L2 flush before each."""
    import torch
    from hybrid_precision_attention_b200 import hq, synth
    lay = synth.planted_layer(0, B, HQ, HKV, L)
    k_d, v_d, qt_d = [torch.from_numpy(a).cuda() for a in (lay.k, lay.v, lay.q_tail)]
    c = hq.HybridCache(B, HQ, HKV, L + 256, W, RHO_BP)
    hq.hq_select_vlines(c, k_d, qt_d)
    hq.hq_pack_merge(c, k_d, v_d)
    q, k, v = [torch.from_numpy(a).cuda() for a in synth.decode_tokens(1, B, HQ, HKV, 4)]
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    for i in range(4):
        flush.zero_()
        hq.hq_decode_attn(c, q[i], k[i], v[i])
    torch.cuda.synchronize()
    st = c.state()
    assert st["err"] == 0 and st["T"] == L + 4, st
    print("profile-decode ok", st)


def profile_select():
    """Small case for ncu captures: a decode-mode reselection of one 32K layer (prefix install, 64 decode
    steps filling the query buffer, L2 flushed, then hq_select_vlines: two passes and the top-k)."""
    import torch
    from hybrid_precision_attention_b200 import hq, synth
    lay = synth.planted_layer(0, B, HQ, HKV, L)
    k_d, v_d, qt_d = [torch.from_numpy(a).cuda() for a in (lay.k, lay.v, lay.q_tail)]
    c = hq.HybridCache(B, HQ, HKV, L + 256, W, RHO_BP)
    hq.hq_select_vlines(c, k_d, qt_d)
    hq.hq_pack_merge(c, k_d, v_d)
    q, k, v = [torch.from_numpy(a).cuda() for a in synth.decode_tokens(1, B, HQ, HKV, PERIOD)]
    for i in range(PERIOD):
        hq.hq_decode_attn(c, q[i], k[i], v[i])
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    flush.zero_()
    hq.hq_select_vlines(c)
    torch.cuda.synchronize()
    st = c.state()
    assert st["err"] == 0 and st["n_q"] == PERIOD and st["k_sel"] > 0, st
    print("profile-select ok", st)


def profile_prefill():
    """Small case for ncu captures: the hybrid prefill at L=8192 (B=1, Hq=32, Hkv=8), three calls."""
    import torch
    from hybrid_precision_attention_b200 import hq, synth
    Lp = 8192
    lay = synth.planted_layer(2, 1, PF_HQ, PF_HKV, Lp)
    Q = torch.from_numpy(synth.full_queries(2, 1, PF_HQ, PF_HKV, Lp)).cuda()
    k, v = torch.from_numpy(lay.k).cuda(), torch.from_numpy(lay.v).cuda()
    c = hq.HybridCache(1, PF_HQ, PF_HKV, Lp, W, RHO_BP)
    hq.hq_select_vlines(c, k, Q[:, :, Lp - 64:].contiguous())
    torch.cuda.synchronize()
    ws = torch.empty(hq.hq_prefill_workspace_bytes(1, PF_HQ, PF_HKV, Lp), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        hq.hq_prefill_attn(Q, k, v, c.vl_sel, c.state()["k_sel"], W, ws=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].cpu().numpy().view(np.uint32)[0]) == 0
    print("profile-prefill ok")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--profile-decode", action="store_true", help="small case for ncu: 4 decode steps of one 32K layer")
    ap.add_argument("--profile-prefill", action="store_true", help="small case for ncu: 3 prefill calls at L=8192")
    ap.add_argument("--profile-select", action="store_true", help="small case for ncu: one decode-mode reselection at 32K")
    args = ap.parse_args()
    if args.profile_decode:
        profile_decode()
        return
    if args.profile_prefill:
        profile_prefill()
        return
    if args.profile_select:
        profile_select()
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
