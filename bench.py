"""Benchmark of the TurboQuant hot path on B200: encode -> score -> top-k.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config kv|decode|tiny|search|larged]
                    [--impl ours|reference]

One step = one pass of the whole path over one batch of synthetic input:
tq_encode of every vector, then the estimates of the queries against all
codes and their top-10 (one tq_score_topk call when a config has both, which
transforms and scores the queries once; else tq_score or tq_topk alone).
Default workload ("kv"): KV-cache keys
bf16 [8 KV heads, 32768 tokens, 128], b = 4, with 4 decode query heads per KV
head (GQA 4:1, 32 query heads).  Inputs sit in HBM before the timed region;
L2 (126 MB) is flushed by writing a 256 MB buffer between timed steps.

Multi-GPU (torchrun, one rank per GPU): weak scaling -- every rank encodes and
scores its own independent batch (the vectors are independent problems, so
there is no data-path collective); the time is the max over ranks.

--impl reference times the plain CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "tq_encode Mvec/s and tq_score scores/s over packed codes; HBM GB/s vs B200 peak"

CONFIGS = {
    # name: G groups, n vectors/group, d, b, input kind, queries per group, k
    "kv": dict(G=8, n=32768, d=128, b=4, x="kv", nq=4, q="kv", k=10, score=True, topk=True,
               desc="KV keys bf16 [1,8,32768,128] (4 outlier channels x20 per head), b=4; "
                    "decode queries bf16 32 heads GQA 4:1"),
    "kv_mse": dict(G=8, n=32768, d=128, b=4, x="kv", nq=4, q="kv", k=10, score=True, topk=True,
                   variant="mse",
                   desc="KV keys bf16 [1,8,32768,128] as kv, MSE-only variant (4-bit Lloyd-Max "
                        "index, no QJL); decode queries bf16 32 heads GQA 4:1"),
    "decode": dict(G=8, n=131072, d=128, b=4, x="kv", nq=4, q="kv", k=10, score=True, topk=True,
                   desc="decode attention logits, Llama-3.1-8B-shaped: 32 q heads / 8 KV heads, "
                        "head_dim 128, context 131072, bf16, b=4"),
    "tiny": dict(G=1, n=4096, d=128, b=4, x="rows", nq=64, q="gauss", k=10, score=True, topk=True,
                 desc="tiny: 4096 x 128 fp32 rows (norms U[0.5,2]), 64 queries, b=4"),
    "search": dict(G=1, n=1_000_000, d=1536, b=4, x="unit", nq=1024, q="unit", k=10, score=False,
                   topk=True, desc="embedding search: 1e6 x 1536 fp32 unit rows, 1024 queries, "
                                   "b=4, top-10"),
    "larged": dict(G=1, n=1_000_000, d=3072, b=4, x="rows", nq=256, q="gauss", k=10, score=True,
                   topk=True, desc="large-d: 1e6 x 3072 fp32 rows (norms U[0.5,2]), 256 queries, "
                                   "b=4"),
}

FFMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # FP32 CUDA-core peak at max SM clock

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the dominant kernel, from one ncu capture of `python bench.py --steps 2
# --warmup 3 --no-cpu-baseline --no-count` (summary under profiles/).  It is
# reported only while the kernel's sources still hash to what was captured.
NCU_TRAFFIC = {
    ("kv", "k_encode_tc"): {
        "sources": ["kv_cache_embedding_b200/csrc/tq_encode_tc.cu"],
        "sha1": "d0fba32e71c4e1608d47cd281935347fa9eba732",
        "bytes": 68254208 + 4477696,
    },
}


def ncu_traffic(config, kernel):
    import hashlib
    rec = NCU_TRAFFIC.get((config, kernel))
    if rec is None:
        return None
    h = hashlib.sha1()
    for rel in rec["sources"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return rec["bytes"] if h.hexdigest() == rec["sha1"] else None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"],
                    bf16_sus=p.get("bf16_tflops_sustained", p["bf16_tflops"]), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ---------------------------------------------------------------- inputs
def make_inputs(cfg, device, seed_offset=0, max_rows=None):
    import synth
    G, n, d, nq = cfg["G"], cfg["n"], cfg["d"], cfg["nq"]
    if max_rows is not None and n > max_rows:
        G, n = 1, max_rows
    s = 1 + 100 * seed_offset
    if cfg["x"] == "kv":
        x = synth.kv_keys(G, n, d, seed=s, device=device)
    elif cfg["x"] == "unit":
        x = synth.gaussian_rows(G * n, d, seed=s, device=device, unit=True).reshape(G, n, d)
    else:
        x = synth.gaussian_rows(G * n, d, seed=s, device=device).reshape(G, n, d)
    if cfg["q"] == "kv":
        q = synth.kv_queries(G * nq, G, d, seed=s + 1, device=device, key_seed=s)
    elif cfg["q"] == "unit":
        q = synth.gaussian_rows(G * nq, d, seed=s + 1, device=device, unit=True).reshape(G, nq, d)
    else:
        q = synth.gaussian_rows(G * nq, d, seed=s + 1, device=device,
                                norm_range=None).reshape(G, nq, d)
    return x.contiguous(), q.contiguous()


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every 5 ms in a
    background thread through NVML (the library behind nvidia-smi); falls back
    to `nvidia-smi -lms 50` when NVML is unavailable."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device):
        self.device = device
        self.rows = []        # (time, sm_mhz, sm_max_mhz, reason names)
        self.proc = None
        self.t = None
        self.stop_ev = threading.Event()
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(
                uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            idx = self.device.index if self.device.index is not None else 0
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                idx = int(vis.split(",")[idx])
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))

            def loop():
                while not self.stop_ev.is_set():
                    try:
                        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        bits = int(get_reasons(h))
                    except Exception:
                        break
                    names = [n for b, n in self.REASONS.items() if bits & b]
                    self.rows.append((time.time(), sm, mx, names))
                    self.stop_ev.wait(0.005)

            self.source = "nvml 5 ms"
            self.t = threading.Thread(target=loop, daemon=True)
            self.t.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device.index or 0), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.source = "nvidia-smi 50 ms"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

        def read():
            for line in self.proc.stdout:
                r = [c.strip() for c in line.split(",")]
                if len(r) < 9 or not r[1].replace(".", "").isdigit():
                    continue
                self.rows.append((time.time(), float(r[1]),
                                  float(r[2]) if r[2].replace(".", "").isdigit() else None,
                                  [names[i] for i in range(4) if r[5 + i] == "Active"]))

        self.t = threading.Thread(target=read, daemon=True)
        self.t.start()

    def wait_first(self, timeout=5.0):
        """Block until the first sample is in (so the timed region is covered)."""
        t_end = time.time() + timeout
        while not self.rows and time.time() < t_end and (self.t and self.t.is_alive()):
            time.sleep(0.01)

    def stop(self):
        self.stop_ev.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.t:
            self.t.join(timeout=2)

    def summary(self, t0, t1):
        rows = [r for r in self.rows if t0 <= r[0] <= t1]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "source": self.source}
        sm = [r[1] for r in rows]
        mx = [r[2] for r in rows if r[2] is not None]
        reasons = sorted({n for r in rows for n in r[3]})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "source": self.source,
                "window": "timed region"}


# ---------------------------------------------------------------- ranks
def rank_max(dist, values, device):
    """Max over ranks of each value: a multi-GPU time is the slowest rank's."""
    if dist is None:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(units_per_rank, world, steps, total_ms):
    """Whole-job Mvec/s: the units every rank processed over `steps` steps,
    divided by the (max-over-ranks) device time."""
    return units_per_rank * world * steps / (total_ms / 1e3) / 1e6


# ---------------------------------------------------------------- our arm
class Step:
    """One pass of the hot path with preallocated outputs and workspaces."""

    def __init__(self, tq, cfg, x, q):
        import kv_cache_embedding_b200 as K
        self.K = K
        self.cfg = cfg
        self.tq = tq
        self.x, self.q = x, q
        G, n, d, nq, k = cfg["G"], cfg["n"], cfg["d"], cfg["nq"], cfg["k"]
        dev = x.device
        self.codes = K.Codes(torch.empty(G, n, tq.words, dtype=torch.int32, device=dev),
                             torch.empty(G, n, dtype=torch.float32, device=dev),
                             torch.empty(G, n, dtype=torch.float32, device=dev))
        self.scores = torch.empty(G, nq, n, dtype=torch.float32, device=dev) if cfg["score"] else None
        self.topk = (torch.empty(G, nq, k, dtype=torch.float32, device=dev),
                     torch.empty(G, nq, k, dtype=torch.int64, device=dev)) if cfg["topk"] else None
        B = K.binding
        # scores and top-k together: one call (tq_score_topk) scores once
        self.combined = bool(cfg["score"] and cfg["topk"])
        need = max(B.tq_workspace_bytes(B.TQ_OP_ENCODE, d, cfg["b"], G, n, nq, k),
                   B.tq_workspace_bytes(B.TQ_OP_SCORE, d, cfg["b"], G, n, nq, k),
                   B.tq_workspace_bytes(B.TQ_OP_TOPK, d, cfg["b"], G, n, nq, k),
                   B.tq_workspace_bytes(B.TQ_OP_SCORE_TOPK, d, cfg["b"], G, n, nq, k))
        tq.ws.get(need)
        self.ev = None

    def outputs(self):
        """Every result tensor of a step (what an end-to-end caller reads back)."""
        out = [self.codes.codes, self.codes.xnorm, self.codes.rnorm]
        if self.scores is not None:
            out.append(self.scores)
        if self.topk is not None:
            out += list(self.topk)
        return out

    def run(self, events=None):
        """events: optional list of 4 CUDA events recorded between the calls
        (encode | score | top-k; with the combined call the score interval
        holds tq_score_topk and the top-k interval is empty)."""
        tq = self.tq
        if events:
            events[0].record()
        tq.encode(self.x, out=self.codes)
        if events:
            events[1].record()
        if self.combined:
            tq.score_topk(self.codes, self.q, self.cfg["k"], scores_out=self.scores,
                          topk_out=self.topk)
            if events:
                events[2].record()
                events[3].record()
            return
        if self.scores is not None:
            tq.score(self.codes, self.q, out=self.scores)
        if events:
            events[2].record()
        if self.topk is not None:
            tq.topk(self.codes, self.q, self.cfg["k"], out=self.topk)
        if events:
            events[3].record()


def count_launches(step):
    """Kernels launched by one step, counted with the CUDA profiler (CUPTI)."""
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step.run()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type.name == "CUDA"
                 and not e.name.startswith(("Memcpy", "Memset", "cudaMem"))]
        ours = [nm.replace("(anonymous namespace)::", "") for nm in names if "tq::" in nm]
        return len(ours), sorted({nm.split("(")[0] for nm in ours})
    except Exception as e:  # profiler unavailable
        return None, [f"profiler unavailable: {e}"]


def alg_bytes_flops(cfg):
    G, n, d, b, nq, k = cfg["G"], cfg["n"], cfg["d"], cfg["b"], cfg["nq"], cfg["k"]
    esz = 2 if cfg["x"] == "kv" else 4
    rec = b * d // 8 + 8
    enc_bytes = G * n * (d * esz + rec)
    # two d x d products per vector (rotation, QJL projection); one for MSE-only
    enc_flops = (2.0 if cfg.get("variant", "prod") == "mse" else 4.0) * d * d * G * n
    score_bytes = G * n * rec + G * nq * n * 4
    score_flops = 4.0 * d * G * n * nq
    topk_bytes = G * n * rec + G * nq * k * 12
    return dict(enc_bytes=enc_bytes, enc_flops=enc_flops, score_bytes=score_bytes,
                score_flops=score_flops, topk_bytes=topk_bytes, rec=rec)


def run_ours(args, cfg, rank, world, dist):
    import kv_cache_embedding_b200 as K
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    x, q = make_inputs(cfg, dev, seed_offset=rank)
    tq = K.TurboQuant(cfg["d"], cfg["b"], seed=0, groups=cfg["G"], device=dev,
                      variant=cfg.get("variant", "prod"))
    step = Step(tq, cfg, x, q)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    nlaunch, kernel_names = count_launches(step) if not args.no_count else (None, [])
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    # The step as one CUDA graph (the same public calls, captured once): its
    # replays are the timed steps.  Per-call times come from a second timed
    # pass of plain stream launches.
    graph = None
    if not args.no_graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step.run()
            torch.cuda.synchronize()
            for _ in range(args.warmup):
                graph.replay()
            torch.cuda.synchronize()
        except Exception as e:  # capture unsupported: plain launches
            print(f"graph capture failed ({e}); timing plain launches", file=sys.stderr)
            graph = None
            torch.cuda.synchronize()
    sampler = ClockSampler(dev)
    sampler.start()
    sampler.wait_first()
    gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for i in range(args.steps):
        flush.zero_()
        if graph is not None:
            gev[i][0].record()
            graph.replay()
            gev[i][1].record()
        else:
            step.run(evs[i])
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    t1 = time.time()
    if graph is not None:  # per-call breakdown, plain launches
        for i in range(args.steps):
            flush.zero_()
            step.run(evs[i])
        torch.cuda.synchronize()
    time.sleep(0.3)
    sampler.stop()
    enc = [e[0].elapsed_time(e[1]) for e in evs]
    sco = [e[1].elapsed_time(e[2]) for e in evs]
    tpk = [e[2].elapsed_time(e[3]) for e in evs]
    if graph is not None:
        tot_ms = sum(e[0].elapsed_time(e[1]) for e in gev)
    else:
        tot_ms = sum(e[0].elapsed_time(e[3]) for e in evs)
    tot_ms, se, ss, st = rank_max(dist, [tot_ms, sum(enc), sum(sco), sum(tpk)], dev)
    K_ = args.steps
    ms_step = tot_ms / K_
    units = cfg["G"] * cfg["n"] * world
    value = job_throughput(cfg["G"] * cfg["n"], world, K_, tot_ms)

    # e2e: every step copies its inputs from pinned host memory to the device,
    # runs the same three public calls and copies every result back to pinned
    # host memory.  Two buffer sets and one stream per copy direction let the
    # copies of neighbouring steps overlap the compute (and each other).
    xh = x.cpu().pin_memory()
    qh = q.cpu().pin_memory()
    bufs = []
    for _ in range(2):
        xd, qd = torch.empty_like(x), torch.empty_like(q)
        stp = Step(tq, cfg, xd, qd)
        host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in stp.outputs()]
        bufs.append((xd, qd, stp, host))
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(m):
        start = torch.cuda.Event()
        start.record()
        for s_ in (s_in, s_c, s_out):
            s_.wait_event(start)
        for i in range(m):
            j = i % 2
            xd, qd, stp, host = bufs[j]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_c[j])  # step i-2 has finished reading xd, qd
                xd.copy_(xh, non_blocking=True)
                qd.copy_(qh, non_blocking=True)
                ev_in[j].record(s_in)
            with torch.cuda.stream(s_c):
                s_c.wait_event(ev_in[j])
                if i >= 2:
                    s_c.wait_event(ev_out[j])  # step i-2's results are on the host
                stp.run()
                ev_c[j].record(s_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[j])
                for h, t in zip(host, stp.outputs()):
                    h.copy_(t, non_blocking=True)
                ev_out[j].record(s_out)
        cur = torch.cuda.current_stream()
        for s_ in (s_in, s_c, s_out):
            cur.wait_stream(s_)

    e2e_run(max(2, min(args.warmup, 3)))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(2, min(args.steps, 20))
    if dist:
        dist.barrier()
    e0.record()
    e2e_run(e2e_steps)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = rank_max(dist, [e0.elapsed_time(e1) / e2e_steps], dev)[0]
    h2d = xh.numel() * xh.element_size() + qh.numel() * qh.element_size()
    d2h = sum(t.numel() * t.element_size() for t in bufs[0][3])

    ab = alg_bytes_flops(cfg)
    pk = peaks()
    enc_ms = se / K_
    score_ms = ss / K_ if cfg["score"] else None
    topk_ms = st / K_ if cfg["topk"] else None
    # dominant kernel: the encode call.  For d = 128 bf16 keys it is one fused
    # tcgen05 kernel: the rotation takes 2 fp16 passes (exact fp16 keys times
    # two pieces of Pi), the QJL product 3, so its peak is the measured 16-bit
    # peak / 2.5 (the mean pass count over the two equal-sized products).
    ach = ab["enc_flops"] / (enc_ms / 1e3) / 1e12
    mse = cfg.get("variant", "prod") == "mse"
    tc = cfg["d"] == 128 and cfg["x"] == "kv" and not mse
    if cfg["d"] >= 256:
        # split-precision tcgen05 GEMMs: the rotation takes 3 16-bit passes for
        # bf16 inputs (one exact piece) and 6 for fp32 inputs, the QJL product 6
        p_rot = 3 if cfg["x"] == "kv" else 6
        passes = [p_rot] if mse else [p_rot, 6]
        peak = pk["bf16"] * len(passes) / sum(passes)
        roofline = {"bound": "tensor", "achieved": round(ach, 2), "peak": round(peak, 1),
                    "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": None,
                    "alg_bytes": ab["enc_bytes"],
                    "kernel": "k_gemm_tc (tq_encode: rotation and QJL as split-bf16 tcgen05 "
                              "GEMMs) + k_quantize + k_pack",
                    "peak_source": f"measured bf16 burst (MEASURED_PEAKS.json) / "
                                   f"{sum(passes) / len(passes):g} passes (mean over the products)",
                    "hbm_gbs": round(ab["enc_bytes"] / enc_ms / 1e6, 1),
                    "hbm_frac": round(ab["enc_bytes"] / enc_ms / 1e6 / pk["hbm"], 4)}
    elif tc:
        peak = pk["bf16"] / 2.5
        roofline = {"bound": "tensor", "achieved": round(ach, 2), "peak": round(peak, 1),
                    "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                    "traffic": ncu_traffic(args.config, "k_encode_tc"),
                    "alg_bytes": ab["enc_bytes"],
                    "kernel": "k_encode_tc (tq_encode: rotation (2 fp16 passes) + QJL (3) on "
                              "tcgen05, fused epilogue)",
                    "peak_source": "measured bf16 burst (MEASURED_PEAKS.json) / 2.5 passes "
                                   "(fp16 = bf16 rate)",
                    "frac_of_3xtf32_fp32_equivalent": round(ach / (pk["bf16"] * 0.5 / 3.0), 4),
                    "hbm_gbs": round(ab["enc_bytes"] / enc_ms / 1e6, 1),
                    "hbm_frac": round(ab["enc_bytes"] / enc_ms / 1e6 / pk["hbm"], 4)}
    else:
        roofline = {"bound": "alu", "achieved": round(ach, 3), "peak": round(FFMA_PEAK_TFLOPS, 1),
                    "unit": "TFLOP/s", "frac": round(ach / FFMA_PEAK_TFLOPS, 4), "traffic": None,
                    "kernel": "tq_encode portable path (fp32 FFMA GEMMs)",
                    "peak_source": "derived: 148 SM x 128 FP32 lanes x 2 x 1965 MHz"}
    out = {
        "metric": METRIC, "value": round(value, 4), "unit": "Mvec/s", "n_gpus": world,
        "steps": K_, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; shapes of the pages' KV-cache / embedding workloads)",
        "config": {"workload": f"{args.config}: {cfg['desc']}", "G": cfg["G"], "n": cfg["n"],
                   "d": cfg["d"], "b": cfg["b"], "queries_per_group": cfg["nq"], "k": cfg["k"],
                   "l2": "flushed (256 MB write) between timed steps",
                   "launch": "CUDA graph of the step" if graph is not None else "stream launches",
                   "parallelism": f"dp{world} (independent batches per GPU)"},
        "encode": {"ms": round(enc_ms, 5),
                   "mvec_s": round(cfg["G"] * cfg["n"] / enc_ms / 1e3, 3),
                   "gbs": round(ab["enc_bytes"] / enc_ms / 1e6, 2),
                   "hbm_frac": round(ab["enc_bytes"] / enc_ms / 1e6 / pk["hbm"], 4)},
        "roofline": roofline,
        "e2e": {"value": round(units / e2e_ms / 1e3, 4), "unit": "Mvec/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": (nlaunch * K_) if nlaunch is not None else None,
        "gpu_launches_per_step": nlaunch,
        "kernels": kernel_names,
        "clocks": sampler.summary(t0, t1),
        "peaks": pk,
    }
    if step.combined:
        # tq_score_topk: the score matrix and the top-k lists from one scoring pass
        sg = ab["score_bytes"] / score_ms / 1e6
        out["score_topk"] = {"ms": round(score_ms, 5),
                             "scores_s": round(cfg["G"] * cfg["nq"] * cfg["n"] / score_ms * 1e3, 1),
                             "gbs": round(sg, 2), "hbm_frac": round(sg / pk["hbm"], 4),
                             "call": "tq_score_topk (scores written + top-k of the same pass)"}
    else:
        if score_ms is not None:
            sg = ab["score_bytes"] / score_ms / 1e6
            out["score"] = {"ms": round(score_ms, 5),
                            "scores_s": round(cfg["G"] * cfg["nq"] * cfg["n"] / score_ms * 1e3, 1),
                            "gbs": round(sg, 2), "hbm_frac": round(sg / pk["hbm"], 4)}
        if topk_ms is not None:
            out["topk"] = {"ms": round(topk_ms, 5),
                           "scores_s": round(cfg["G"] * cfg["nq"] * cfg["n"] / topk_ms * 1e3, 1)}
    if args.config == "decode" and rank == 0:
        out["fp32_baseline"] = fp32_baseline(cfg, x, q, flush, args)
        out["attention"] = attention_decode_time(cfg, x, q, flush, args)
    return out


def attention_decode_time(cfg, x, q, flush, args):
    """Decode attention over the same keys (b-bit inner-product records) and
    seeded values (4-bit MSE-only records): one tq_attention_decode call per
    timed iteration, L2 flushed in between.  Not part of the step."""
    import kv_cache_embedding_b200 as K
    import synth
    G, n, d = cfg["G"], cfg["n"], cfg["d"]
    tk = K.TurboQuant(d, cfg["b"], seed=0, groups=G, device=x.device)
    tv = K.TurboQuant(d, 4, seed=1, groups=G, device=x.device, variant="mse")
    kc = tk.encode(x)
    vc = tv.encode(synth.kv_keys(G, n, d, seed=5, device=x.device))
    out = tk.attention_decode(kc, tv, vc, q)
    for _ in range(3):
        tk.attention_decode(kc, tv, vc, q, out=out)
    ts = []
    for _ in range(max(3, min(args.steps, 50))):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        tk.attention_decode(kc, tv, vc, q, out=out)
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    ms = sum(ts) / len(ts)
    byts = (kc.codes.numel() * 4 + kc.xnorm.numel() * 8 + vc.codes.numel() * 4 +
            vc.xnorm.numel() * 4 + q.numel() * q.element_size() + out.numel() * 4)
    return {"ms": round(ms, 5), "gbs": round(byts / ms / 1e6, 1),
            "values": "4-bit MSE-only records (seeded keys-like rows)", "scale": "1/sqrt(d)"}


def fp32_baseline(cfg, x, q, flush, args):
    """Unquantized fp32 keys: logits kernel time vs tq_score on packed codes."""
    import kv_cache_embedding_b200 as K
    keys = x.float()
    out = torch.empty(cfg["G"], cfg["nq"], cfg["n"], dtype=torch.float32, device=x.device)
    for _ in range(3):
        K.logits_fp32(keys, q, out)
    ts = []
    for _ in range(max(3, min(args.steps, 50))):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        K.logits_fp32(keys, q, out)
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    ms = sum(ts) / len(ts)
    byts = keys.numel() * 4 + out.numel() * 4
    return {"ms": round(ms, 5), "gbs": round(byts / ms / 1e6, 1)}


# ---------------------------------------------------------------- oracle arm
def oracle_sample(cfg, target_s=10.0, max_units=None):
    """Run the oracle's encode -> score -> top-k on a bounded sample of the
    workload; returns (vectors, seconds, description)."""
    import numpy as np
    from oracle import oracle as O
    G, n, d, b, nq, k = cfg["G"], cfg["n"], cfg["d"], cfg["b"], cfg["nq"], cfg["k"]
    x, q = make_inputs(cfg, "cpu", max_rows=65536)
    n = min(n, x.shape[1])
    mse = cfg.get("variant", "prod") == "mse"
    # one group's parameters (built outside the timing)
    params = O.MseParams(d, b, 0) if mse else O.Params(d, b, 0)

    def run(rows):
        xs = x[0, :rows].to(torch.float64).numpy()
        qs = q[0].to(torch.float64).numpy()
        t = time.perf_counter()
        if mse:
            codes, xn, rn = O.mse_encode(params, xs)
            s = O.mse_score(params, codes, xn, qs)
        else:
            codes, xn, rn = O.encode(params, xs)
            s = O.score(params, codes, xn, rn, qs)
        O.topk(s, min(k, rows))
        return time.perf_counter() - t

    rows = min(n, 256)
    dt = run(rows)
    cap = max_units or n
    while dt < target_s / 4 and rows < min(n, cap):
        rows = min(n, cap, rows * 4)
        dt = run(rows)
    return rows, dt, (f"{rows} of the {G * n} vectors (group 0), oracle encode + score of "
                      f"{nq} queries + top-{k}, extrapolated per vector")


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, cfg):
    steps = []
    for i in range(args.warmup + args.steps):
        rows, dt, desc = oracle_sample(cfg, target_s=max(0.5, 8.0 / max(args.steps, 1)))
        if i >= args.warmup:
            steps.append((rows, dt))
    rows = sum(r for r, _ in steps)
    secs = sum(t for _, t in steps)
    value = rows / secs / 1e6
    cores = int(os.environ.get("OMP_NUM_THREADS", cpu_cores()))
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mvec/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / len(steps) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.config}: {cfg['desc']}", "G": cfg["G"], "n": cfg["n"],
                   "d": cfg["d"], "b": cfg["b"]},
        "cpu_baseline": {"value": value, "unit": "Mvec/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "Mvec/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="kv", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time plain stream launches instead of replays of the step's CUDA graph")
    ap.add_argument("--no-count", action="store_true",
                    help="skip the profiler-based launch count (for runs under ncu)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = CONFIGS[args.config]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, cfg)))
        return 0

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as td
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = td
    out = run_ours(args, cfg, rank, world, dist)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows, dt, desc = oracle_sample(cfg, target_s=10.0)
        out["cpu_baseline"] = {"value": rows / dt / 1e6, "unit": "Mvec/s",
                               "cores": int(os.environ.get("OMP_NUM_THREADS", cpu_cores())),
                               "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(out))
    if dist:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
