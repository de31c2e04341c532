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


def decode_bytes(n_packed, n_vl, T, b=B, hkv=HKV, hq=HQ):
    """Algorithmic bytes of one decode step (all kv heads) at the given state (before the step):
    packed positions outside the VL set at 160 B, FP16 rows (VL, ring, new token) at 512 B."""
    fp16_rows = n_vl + (T + 1 - n_packed)
    per_head = (n_packed - n_vl) * 160 + fp16_rows * 512
    return b * hkv * per_head + 2 * b * hq * D * 2


def period_bytes(T0, b=B, hkv=HKV, hq=HQ, tokens=PERIOD):
    """Algorithmic decode bytes of `tokens` decode steps starting right after a merge at length T0."""
    n_packed = T0 - W
    n_vl = k_of(n_packed, RHO_BP)
    return sum(decode_bytes(n_packed, n_vl, T0 + t, b, hkv, hq) for t in range(tokens))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def load_extra_peaks():
    """Peaks this repository measured on the same GPUs (the committed record
    profiles/peaks_b200.json, written by `bench.py --measure-peaks`): the dense
    e4m3 tensor peak and the read-only HBM streaming ceiling."""
    p = os.path.join(ROOT, "profiles", "peaks_b200.json")
    if os.path.exists(p):
        return json.load(open(p))
    return {}


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


def run_prefill(dev, reps=5, warmup=2, qk_format=0):
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
    ws = torch.empty(hq.hq_prefill_workspace_bytes(1, PF_HQ, PF_HKV, PF_L, vl.shape[2]), dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        hq.hq_prefill_attn(q_d, k_d, v_d, vl, n_vl, W, out=out, ws=ws, qk_format=qk_format)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        hq.hq_prefill_attn(q_d, k_d, v_d, vl, n_vl, W, out=out, ws=ws, qk_format=qk_format)
    e1.record()
    torch.cuda.synchronize()
    err = int(ws[:4].cpu().numpy().view(np.uint32)[0])
    assert err == 0, err
    ms = e0.elapsed_time(e1) / reps
    flops = prefill_flops(PF_L, PF_HQ)
    tflops = flops / (ms * 1e-3) / 1e12
    bf16, kind = load_bf16_peak()
    extra = load_extra_peaks()
    key, name = ("int8_tops", "INT8") if qk_format == 1 else ("fp8_e4m3_tflops", "e4m3")
    if key in extra:
        fp8, fp8_kind = float(extra[key]), f"measured {name} GEMM (profiles/peaks_b200.json)"
    else:
        fp8, fp8_kind = 2.0 * bf16, f"{kind} bf16 x 2 (nominal fp8/bf16 ratio)"
    mixed = 1.0 / (0.5 / fp8 + 0.5 / bf16)
    fmt = "INT8 Q.K + FP16 P.V" if qk_format == 1 else "e4m3 Q.K (P.V on f16 with e4m3 V values)"
    return {"workload": f"causal hybrid prefill, B=1, L=32768, Hq=32, Hkv=8, D=128, W=128, rho=5% ({n_vl} lines per kv head), "
                        f"quantised tiles {fmt}",
            "ms": ms, "tflops": tflops, "calls": reps,
            "roofline": {"kernel": "prefill (pre-pass + prefill_kernel)", "bound": "tensor", "achieved": tflops,
                         "peak": fp8, "unit": "TFLOP/s", "frac": tflops / fp8, "traffic": None,
                         "peak_kind": fp8_kind,
                         "mixed_ceiling": mixed,
                         "note": f"QK of quantised tiles on {name} ({name} rate), P.V on f16 (bf16 rate): half the "
                                 "flops at each rate, so the ceiling of this mix is the mixed_ceiling figure"}}


def decode_traffic_record(bytes_per_launch):
    """DRAM traffic of a decode launch from the committed ncu record
    (profiles/decode_kernel_32k.traffic.json: the captured launch's T, its
    algorithmic bytes and its DRAM read + write bytes), scaled to this run's
    average launch by algorithmic bytes (the traffic grows with the positions
    scanned).  None unless the record was taken on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "decode_kernel_32k.traffic.json")
    if not os.path.exists(p):
        return None, None
    rec = json.load(open(p))
    if rec.get("sources_sha256") != kernel_sources_sha("decode.cu"):
        return None, rec
    scaled = rec["dram_bytes"] * bytes_per_launch / rec["algorithmic_bytes"]
    return scaled, rec


def kernel_sources_sha(*names):
    """sha256 over the code of the named kernel sources plus the shared device
    header: comments removed and whitespace collapsed, so a comment-only edit
    keeps a record taken on the same code."""
    h = hashlib.sha256()
    for n in list(names) + ["common.cuh"]:
        src = open(os.path.join(ROOT, "hybrid_precision_attention_b200", "csrc", n)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(re.sub(r"\s+", " ", src).strip().encode())
    return h.hexdigest()


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
    cap = L + PERIOD * (n_steps_total + 8) + 256   # + the eager period and two e2e legs of up to 3 periods

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
    # reselection (sel_pass<0>, sel_pass<1>, the top-k) and a staging merge
    # (merge_gather_kernel, vl_install_kernel)
    launches_per_step = PERIOD * COPIES + COPIES * (3 + 2)

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
    traffic, trec = decode_traffic_record(bytes_per_launch)
    extra = load_extra_peaks()
    roof = {"kernel": "decode_kernel", "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": traffic, "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json)",
            "avg_launch_us": dec_avg_us, "algorithmic_bytes_per_launch": bytes_per_launch,
            "traffic_record": trec}
    if "hbm_read_gbs" in extra:
        roof["read_ceiling_gbs"] = float(extra["hbm_read_gbs"])
        roof["frac_of_read_ceiling"] = achieved / float(extra["hbm_read_gbs"])

    # end-to-end leg: the public API with host buffers, copies inside the timed region.
    # Each step copies its inputs (every token's q, k, v for every layer copy,
    # one pinned host buffer) host -> device in one transfer, runs the period
    # (the decode steps, then the selections and merges) and copies every
    # output back in one transfer.  The headline figure replays that step
    # from a CUDA graph captured through the public API (how a serving loop
    # drives it: the lengths are device-resident); the same step issued
    # eagerly from Python is reported beside it.
    e2e = None
    if not args.no_e2e:
        nq_, nk_ = B * HQ * D, B * HKV * D
        row = nq_ + 2 * nk_
        inh = torch.empty((PERIOD, COPIES, row), dtype=torch.float16).pin_memory()
        for ci in range(COPIES):
            inh[:, ci, :nq_] = torch.from_numpy(qn).reshape(PERIOD, nq_)
            inh[:, ci, nq_:nq_ + nk_] = torch.from_numpy(kn).reshape(PERIOD, nk_)
            inh[:, ci, nq_ + nk_:] = torch.from_numpy(vn).reshape(PERIOD, nk_)
        outh = torch.empty((PERIOD, COPIES, B, HQ, D), dtype=torch.float16).pin_memory()
        ind = torch.empty((PERIOD, COPIES, row), dtype=torch.float16, device=dev)
        outd = torch.empty((PERIOD, COPIES, B, HQ, D), dtype=torch.float16, device=dev)
        n_e2e = max(1, min(args.steps, 3))

        def e2e_step():
            ind.copy_(inh, non_blocking=True)
            for tt in range(PERIOD):
                for ci, c in enumerate(caches):
                    r = ind[tt, ci]
                    hq.hq_decode_attn(c, r[:nq_].view(B, HQ, D), r[nq_:nq_ + nk_].view(B, HKV, D),
                                      r[nq_ + nk_:].view(B, HKV, D), out=outd[tt, ci], stream=stream)
            maint_block()
            outh.copy_(outd, non_blocking=True)

        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e, stream=stream):
            e2e_step()

        def timed(run):
            T_e = caches[0].state()["T"]
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(n_e2e):
                    run()
                    stream.synchronize()   # the step's results are on the host
                e1.record(stream)
            torch.cuda.synchronize()
            ms_max, nbytes = aggregate_ranks(e0.elapsed_time(e1),
                                             sum(period_bytes(T_e + PERIOD * i) for i in range(n_e2e)) * COPIES, world, dev)
            return nbytes / (ms_max * 1e-3) / 1e9

        v_graph = timed(g_e2e.replay)
        v_eager = timed(e2e_step)
        e2e = {"value": v_graph, "unit": UNIT,
               "h2d_bytes_per_step": PERIOD * COPIES * row * 2,
               "d2h_bytes_per_step": PERIOD * COPIES * out.numel() * 2,
               "steps": n_e2e,
               "api": "hq_decode_attn / hq_select_vlines / hq_pack_merge via the Python binding; the step (its "
                      "inputs copied in from pinned host memory, the period, its outputs copied back) captured "
                      "once in a CUDA graph and replayed",
               "eager_value": v_eager}
        del g_e2e

    prefill = prefill_int8 = None
    if not args.no_prefill:
        prefill = run_prefill(dev)
        prefill_int8 = run_prefill(dev, qk_format=1)

    working_set_mb = COPIES * caches[0].nbytes() / 1e6
    legs = {}
    if not args.no_legs and world == 1:
        for c in caches:
            c._ws.clear()
        del caches
        torch.cuda.empty_cache()
        legs["decode_1k"] = run_small_layer_leg(dev)
        torch.cuda.empty_cache()
        legs["qwen3_8b_36_layers_b16"] = run_multilayer_leg(dev, 36, 16, 32)
        legs["qwen3_32b_64_layers_b32"] = run_multilayer_leg(dev, 64, 32, 64, seed0=900)
        for lg in ("qwen3_8b_36_layers_b16", "qwen3_32b_64_layers_b32"):
            legs[lg]["frac_of_copy_peak"] = legs[lg]["gbs"] / peak
            if "hbm_read_gbs" in extra:
                legs[lg]["frac_of_read_ceiling"] = legs[lg]["gbs"] / float(extra["hbm_read_gbs"])

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu:
        gbs, sec, n, threads, _, _ = oracle_sample(min_seconds=args.cpu_seconds)
        cpu = {"value": gbs, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{n} single decode steps of the 32K layer by the float64 oracle ({sec:.2f} s each); "
                         f"prefix install not timed"}
        if legs:
            g1, s1 = oracle_unit_rate(HQ, 1024, steps=8)
            legs["decode_1k"]["cpu_baseline"] = {"value": s1 * 1e6, "unit": "us per decode step", "cores": threads,
                                                 "kind": "oracle", "sample": "8 single decode steps of the 1K layer"}
            legs["qwen3_8b_36_layers_b16"]["cpu_baseline"] = {
                "value": gbs, "unit": UNIT, "cores": threads, "kind": "oracle",
                "sample": "extrapolated: the 32K layer's single-step oracle rate (one (layer, b) unit of this shape), "
                          "the same bytes per second for all 576 units"}
            g4, s4 = oracle_unit_rate(64, 32768, steps=2)
            legs["qwen3_32b_64_layers_b32"]["cpu_baseline"] = {
                "value": g4, "unit": UNIT, "cores": threads, "kind": "oracle",
                "steps_per_s": 1.0 / (s4 * 64 * 32),
                "sample": f"extrapolated: 2 single decode steps of one (layer, b) unit (Hq=64, Hkv=8, 32K) at "
                          f"{s4:.2f} s each, multiplied by 64 layers x 32 sequences for steps/s"}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "us_per_decode_step": us_per_decode, "pct_of_hbm_peak": 100.0 * value / peak,
            "select_merge_share": sum(mnt_ms) / max(sum(dec_ms) + sum(mnt_ms), 1e-9),
            "config": {"workload": WORKLOAD, "B": B, "Hq": HQ, "Hkv": HKV, "D": D, "prefix": L, "W": W,
                       "rho": RHO_BP / 10000, "layer_copies": COPIES, "decode_tokens_per_step": PERIOD,
                       "l2": f"{COPIES} rotating layer copies, {working_set_mb:.0f} MB working set > 126 MB L2",
                       "parallelism": f"replicas x{world}"},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "prefill": prefill, "prefill_int8_qk": prefill_int8,
            "legs": legs,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": sampler.summary()}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- further workloads

def _events(n):
    import torch
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def run_small_layer_leg(dev, steps=4, copies=72):
    """Decode at a 1K prefix (B=1, Hq=32, Hkv=8): `copies` rotating copies of the
    layer (about 180 MB, larger than L2), one CUDA graph per 64-token period of
    decode launches (one per token and copy) and one for the copies'
    reselection + merge.  Reports microseconds per decode step, with and
    without the amortised reselection + merge."""
    import torch
    from hybrid_precision_attention_b200 import hq, synth
    Ls = 1024
    cap = Ls + PERIOD * (steps + 4) + 256
    lay = synth.planted_layer(7, B, HQ, HKV, Ls)
    k_d, v_d, qt_d = [torch.from_numpy(a).to(dev) for a in (lay.k, lay.v, lay.q_tail)]
    caches = []
    for _ in range(copies):
        c = hq.HybridCache(B, HQ, HKV, cap, W, RHO_BP, device=dev)
        hq.hq_select_vlines(c, k_d, qt_d)
        hq.hq_pack_merge(c, k_d, v_d)
        for op in (hq.OP_SELECT, hq.OP_MERGE, hq.OP_DECODE):
            c.workspace(op)
        caches.append(c)
    qn, kn, vn = synth.decode_tokens(8, B, HQ, HKV, PERIOD)
    q_t, k_t, v_t = [torch.from_numpy(a).to(dev) for a in (qn, kn, vn)]
    out = torch.empty((B, HQ, D), dtype=torch.float16, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def dec():
        for t in range(PERIOD):
            for c in caches:
                hq.hq_decode_attn(c, q_t[t], k_t[t], v_t[t], out=out, stream=stream)

    def mnt():
        for c in caches:
            hq.hq_select_vlines(c, stream=stream)
            hq.hq_pack_merge(c, stream=stream)

    with torch.cuda.stream(stream):
        dec()
        mnt()
    stream.synchronize()
    g_dec, g_mnt = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_dec, stream=stream):
        dec()
    with torch.cuda.graph(g_mnt, stream=stream):
        mnt()
    with torch.cuda.stream(stream):
        for _ in range(2):
            g_dec.replay()
            g_mnt.replay()
    stream.synchronize()
    T0 = caches[0].state()["T"]
    evs = [_events(3) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for i in range(steps):
            evs[i][0].record(stream)
            g_dec.replay()
            evs[i][1].record(stream)
            g_mnt.replay()
            evs[i][2].record(stream)
    torch.cuda.synchronize()
    for c in caches:
        assert c.state()["err"] == 0, c.state()
    dec_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    tot_ms = sum(e[0].elapsed_time(e[2]) for e in evs)
    n = PERIOD * copies * steps
    nbytes = sum(period_bytes(T0 + PERIOD * i) for i in range(steps)) * copies
    return {"workload": f"decode, one layer, B=1, Hq=32, Hkv=8, D=128, prefix {Ls}, rho=5%, W=128; {copies} rotating "
                        f"layer copies ({copies * caches[0].nbytes() / 1e6:.0f} MB > L2); CUDA graphs of 64-token periods",
            "us_per_decode_step": dec_ms * 1e3 / n, "us_per_decode_step_with_select_merge": tot_ms * 1e3 / n,
            "gbs": nbytes / (dec_ms * 1e-3) / 1e9, "periods": steps, "decode_launches": n,
            "select_merge_share": (tot_ms - dec_ms) / tot_ms}


def run_multilayer_leg(dev, layers, b, hq_heads, tokens=8, warm=2, seed0=800):
    """One decode step over every layer of a model-shaped cache held resident
    (prefix 32768, Hkv=8, D=128, rho=5%, W=128, planted generator drawn on the
    device), timed with CUDA events over `tokens` steps replayed from a CUDA
    graph of one step (a decode launch per layer); then one reselection +
    merge of every layer, timed on its own, to give the 64-token period cost."""
    import torch
    from hybrid_precision_attention_b200 import hq, synth
    Ll = 32768
    caches = []
    for layer in range(layers):
        k, v, q_tail, _ = synth.planted_layer_device(seed0 + layer, b, hq_heads, HKV, Ll, dev)
        c = hq.HybridCache(b, hq_heads, HKV, Ll + 128, W, RHO_BP, device=dev)
        hq.hq_select_vlines(c, k, q_tail)
        hq.hq_pack_merge(c, k, v)
        del k, v, q_tail
        c.workspace(hq.OP_DECODE)
        caches.append(c)
    torch.cuda.synchronize()
    for c in caches:
        c._ws.pop(hq.OP_SELECT, None)   # the init-mode selection workspace is sized for a dense prefix
    torch.cuda.empty_cache()
    cache_gb = sum(c.nbytes() for c in caches) / 1e9
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed0 + 99)
    qs = torch.randn((tokens + warm, b, hq_heads, D), generator=gen, device=dev).to(torch.float16)
    ks = torch.randn((tokens + warm, b, HKV, D), generator=gen, device=dev).to(torch.float16)
    vs = torch.randn((tokens + warm, b, HKV, D), generator=gen, device=dev).to(torch.float16)
    q_in = torch.empty((b, hq_heads, D), dtype=torch.float16, device=dev)
    k_in = torch.empty((b, HKV, D), dtype=torch.float16, device=dev)
    v_in = torch.empty((b, HKV, D), dtype=torch.float16, device=dev)
    out = torch.empty((b, hq_heads, D), dtype=torch.float16, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def one_step():
        for c in caches:
            hq.hq_decode_attn(c, q_in, k_in, v_in, out=out, stream=stream)

    def feed(i):
        q_in.copy_(qs[i], non_blocking=True)
        k_in.copy_(ks[i], non_blocking=True)
        v_in.copy_(vs[i], non_blocking=True)

    with torch.cuda.stream(stream):
        feed(0)
        one_step()           # eager: sets function attributes
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one_step()
    with torch.cuda.stream(stream):
        for i in range(1, warm):
            feed(i)
            g.replay()
    stream.synchronize()
    T0 = caches[0].state()["T"]
    evs = _events(2 * tokens)
    with torch.cuda.stream(stream):
        for i in range(tokens):
            feed(warm + i)
            evs[2 * i].record(stream)
            g.replay()
            evs[2 * i + 1].record(stream)
    torch.cuda.synchronize()
    for c in caches:
        st = c.state()
        assert st["err"] == 0 and st["T"] == T0 + tokens, st
    step_ms = [evs[2 * i].elapsed_time(evs[2 * i + 1]) for i in range(tokens)]
    n_packed = Ll - W
    n_vl = k_of(n_packed, RHO_BP)
    nbytes = sum(decode_bytes(n_packed, n_vl, T0 + i, b, HKV, hq_heads) for i in range(tokens)) * layers
    ms = float(np.mean(step_ms))
    # one reselection + merge of every layer (the tokens decoded so far are the buffered queries)
    e0, e1 = _events(2)
    with torch.cuda.stream(stream):
        for c in caches:
            c.workspace(hq.OP_SELECT)
            c.workspace(hq.OP_MERGE)
        e0.record(stream)
        for c in caches:
            hq.hq_select_vlines(c, stream=stream)
            hq.hq_pack_merge(c, stream=stream)
        e1.record(stream)
    torch.cuda.synchronize()
    for c in caches:
        assert c.state()["err"] == 0, c.state()
    mnt_ms = e0.elapsed_time(e1)
    gbs = nbytes / (sum(step_ms) * 1e-3) / 1e9
    res = {"workload": f"{layers} layers resident, B={b}, Hq={hq_heads}, Hkv=8, D=128, prefix 32768, rho=5%, W=128 "
                       f"({cache_gb:.1f} GB of hybrid cache); one decode step over every layer from a CUDA graph",
           "ms_per_step": ms, "steps_per_s": 1e3 / ms, "tokens_per_s": b * 1e3 / ms,
           "gb_per_step": nbytes / tokens / 1e9, "gbs": gbs, "steps": tokens,
           "select_merge_ms_all_layers": mnt_ms,
           "ms_per_step_with_select_merge_amortised": ms + mnt_ms / PERIOD,
           "select_merge_share_of_period": mnt_ms / (PERIOD * ms + mnt_ms)}
    del caches
    torch.cuda.empty_cache()
    return res


def oracle_unit_rate(Hq_, Ls, steps=2):
    """Oracle GB/s on single decode steps of one (layer, b) unit: B=1, Hq_, Hkv=8, prefix Ls."""
    from hybrid_precision_attention_b200 import synth
    from oracle import hybrid
    lay = synth.planted_layer(5, 1, Hq_, HKV, Ls)
    c = hybrid.HybridCacheRef(1, Hq_, HKV, W, RHO_BP, Ls + 64)
    c.init_from_prefix(lay.k, lay.v, lay.q_tail)
    q, k, v = synth.decode_tokens(5, 1, Hq_, HKV, steps)
    tt, bb = 0.0, 0
    for i in range(steps):
        st = (c.n_packed, len(c.vl[0][0]), c.T)
        t0 = time.perf_counter()
        c.decode(q[i], k[i], v[i])
        tt += time.perf_counter() - t0
        bb += decode_bytes(*st, 1, HKV, Hq_)
    return bb / tt / 1e9, tt / steps


def measure_peaks(dev):
    """The dense e4m3 GEMM peak (torch._scaled_mm, 8192^3, per-tensor scales,
    bf16 out; best of 20 by CUDA events) and the read-only HBM ceiling (the
    library's streaming-read helper over 8 GiB, best of 10 at 1..4 CTAs per
    SM).  Prints one JSON line: the record committed as profiles/peaks_b200.json."""
    import torch
    from hybrid_precision_attention_b200 import hq
    n = 8192
    a = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn)
    bt = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=dev)
    for _ in range(5):
        torch._scaled_mm(a, bt, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    best = 1e9
    for _ in range(20):
        e0, e1 = _events(2)
        e0.record()
        torch._scaled_mm(a, bt, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    fp8 = 2.0 * n ** 3 / (best * 1e-3) / 1e12
    del a, bt
    ai = torch.randint(-127, 128, (n, n), device=dev, dtype=torch.int8)
    bi = torch.randint(-127, 128, (n, n), device=dev, dtype=torch.int8).t()
    for _ in range(5):
        torch._int_mm(ai, bi)
    besti = 1e9
    for _ in range(20):
        e0, e1 = _events(2)
        e0.record()
        torch._int_mm(ai, bi)
        e1.record()
        torch.cuda.synchronize()
        besti = min(besti, e0.elapsed_time(e1))
    i8 = 2.0 * n ** 3 / (besti * 1e-3) / 1e12
    del ai, bi
    buf = torch.ones(8 << 30, dtype=torch.uint8, device=dev)
    sink = torch.zeros(4, dtype=torch.int32, device=dev)
    rd = {}
    for cps in (1, 2, 3, 4):
        for _ in range(2):
            hq.hq_diag_stream_read(buf, sink, cps)
        tb = 1e9
        for _ in range(10):
            e0, e1 = _events(2)
            e0.record()
            hq.hq_diag_stream_read(buf, sink, cps)
            e1.record()
            torch.cuda.synchronize()
            tb = min(tb, e0.elapsed_time(e1))
        rd[cps] = buf.numel() / (tb * 1e-3) / 1e9
    best_cps = max(rd, key=rd.get)
    rec = {"fp8_e4m3_tflops": fp8, "fp8_how": f"torch._scaled_mm e4m3 x e4m3 -> bf16, {n}^3 (2 n^3 flops), best of 20, CUDA events",
           "int8_tops": i8, "int8_how": f"torch._int_mm int8 x int8 -> int32, {n}^3 (2 n^3 ops), best of 20, CUDA events",
           "hbm_read_gbs": rd[best_cps], "hbm_read_how": f"hq_diag_stream_read over 8 GiB (16-byte streaming loads, "
                                                         f"{best_cps} CTAs of 512 threads per SM), best of 10, CUDA events",
           "hbm_read_by_ctas_per_sm": rd, "gpu": torch.cuda.get_device_name(dev),
           "when": datetime.datetime.now(datetime.timezone.utc).strftime("%Y-%m-%dT%H:%M:%SZ")}
    print(json.dumps(rec), flush=True)


def ablation_sweep(dev, Ls=8192, Ws=(0, 64, 128, 256, 512), rhos=(0, 100, 250, 500, 1000), steps=4):
    """Accuracy ablation over the window W and the vertical-line ratio rho on
    the planted generator (HyQuant digest, results paragraph: a wider window or
    a higher ratio lowers the prefill error).  For every (W, rho): the hybrid
    prefill's relative L2 error and the hybrid decode's (over `steps` tokens)
    against the same kernels with every key FP16 (W >= L).  One JSON line per
    point."""
    import torch
    from hybrid_precision_attention_b200 import hq, synth
    B_, Hq_, Hkv_ = 1, 32, 8
    lay = synth.planted_layer(3, B_, Hq_, Hkv_, Ls)
    Q = torch.from_numpy(synth.full_queries(3, B_, Hq_, Hkv_, Ls)).to(dev)
    k, v = torch.from_numpy(lay.k).to(dev), torch.from_numpy(lay.v).to(dev)
    qt = Q[:, :, Ls - 64:].contiguous()
    qd, kd, vd = [torch.from_numpy(a).to(dev) for a in synth.decode_tokens(3, B_, Hq_, Hkv_, steps)]
    rel = lambda a, b: float(torch.linalg.vector_norm((a.float() - b.float())) / torch.linalg.vector_norm(b.float()))
    no_vl = torch.zeros((B_, Hkv_, 16), dtype=torch.int32, device=dev)
    exact_pf = hq.hq_prefill_attn(Q, k, v, no_vl, 0, Ls)

    def decode_run(W_, rho_):
        c = hq.HybridCache(B_, Hq_, Hkv_, Ls + steps + 64, W_, rho_, device=dev)
        hq.hq_select_vlines(c, k, qt)
        hq.hq_pack_merge(c, k, v)
        outs = [hq.hq_decode_attn(c, qd[t], kd[t], vd[t]).clone() for t in range(steps)]
        torch.cuda.synchronize()
        assert c.state()["err"] == 0, c.state()
        return c, torch.stack(outs)

    _, exact_dec = decode_run(Ls + 64, 0)
    rows = []
    for W_ in Ws:
        for rho_ in rhos:
            c, dec = decode_run(W_, rho_)
            n_vl = c.state()["n_vl"]
            pf = hq.hq_prefill_attn(Q, k, v, c.vl_pos, n_vl, W_)
            torch.cuda.synchronize()
            row = {"L": Ls, "W": W_, "rho": rho_ / 10000, "lines_per_kv_head": n_vl,
                   "prefill_rel_l2": rel(pf, exact_pf), "decode_rel_l2": rel(dec, exact_dec)}
            rows.append(row)
            print(json.dumps(row), flush=True)
    return rows


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


PROFILE_DECODE_CAPTURED = 2   # the decode launch the ncu capture of --profile-decode selects (-s 2 -c 1)


def write_traffic_record(csv_path):
    """Write profiles/decode_kernel_32k.traffic.json from the raw page of the
    ncu capture of --profile-decode (`ncu -i <report> --page raw --csv`): the
    captured launch's DRAM read + write bytes beside its T and its algorithmic
    bytes, stamped with the kernel sources it was taken on."""
    import csv
    rows = list(csv.reader(open(csv_path)))
    head, units = rows[0], rows[1]
    data = [r for r in rows[2:] if len(r) == len(head) and "decode_kernel" in " ".join(r)]
    assert len(data) == 1, f"expected one decode_kernel launch in {csv_path}, found {len(data)}"
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}

    def metric(name):
        i = head.index(name)
        return float(data[0][i].replace(",", "")) * scale[units[i]]
    rd, wr = metric("dram__bytes_read.sum"), metric("dram__bytes_write.sum")
    T = L + PROFILE_DECODE_CAPTURED
    n_packed = L - W
    rec = {"kernel": "decode_kernel", "workload": f"one decode launch of the 32K layer (B={B}, Hq={HQ}, Hkv={HKV}), "
                                                  f"launch {PROFILE_DECODE_CAPTURED} of --profile-decode, L2 flushed before it",
           "T": T, "n_packed": n_packed, "n_vl": k_of(n_packed, RHO_BP),
           "algorithmic_bytes": decode_bytes(n_packed, k_of(n_packed, RHO_BP), T),
           "dram_read_bytes": rd, "dram_write_bytes": wr, "dram_bytes": rd + wr,
           "command": "ncu --set full --clock-control none -k regex:decode_kernel -s 2 -c 1 -o prof_decode "
                      "python bench.py --profile-decode",
           "sources_sha256": kernel_sources_sha("decode.cu")}
    rec["traffic_over_algorithmic"] = rec["dram_bytes"] / rec["algorithmic_bytes"]
    out = os.path.join(ROOT, "profiles", "decode_kernel_32k.traffic.json")
    json.dump(rec, open(out, "w"), indent=1)
    print(json.dumps(rec))


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
    ws = torch.empty(hq.hq_prefill_workspace_bytes(1, PF_HQ, PF_HKV, Lp, c.vl_sel.shape[2]), dtype=torch.uint8, device="cuda")
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
    ap.add_argument("--no-legs", action="store_true", help="skip the 1K, 36-layer and 64-layer decode workloads")
    ap.add_argument("--measure-peaks", action="store_true", help="measure the e4m3 GEMM peak and the read-only HBM ceiling")
    ap.add_argument("--sweep", action="store_true", help="accuracy ablation over W and rho on the planted generator")
    ap.add_argument("--profile-decode", action="store_true", help="small case for ncu: 4 decode steps of one 32K layer")
    ap.add_argument("--profile-prefill", action="store_true", help="small case for ncu: 3 prefill calls at L=8192")
    ap.add_argument("--profile-select", action="store_true", help="small case for ncu: one decode-mode reselection at 32K")
    ap.add_argument("--traffic-record", metavar="CSV", help="write the decode DRAM-traffic record from the raw-page csv "
                                                           "of the --profile-decode ncu capture")
    args = ap.parse_args()
    if args.traffic_record:
        write_traffic_record(args.traffic_record)
        return
    if args.profile_decode:
        profile_decode()
        return
    if args.profile_prefill:
        profile_prefill()
        return
    if args.profile_select:
        profile_select()
        return
    if args.measure_peaks:
        import torch
        measure_peaks(torch.device("cuda", 0))
        return
    if args.sweep:
        import torch
        ablation_sweep(torch.device("cuda", 0))
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
