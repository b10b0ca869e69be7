"""Benchmark of the TurboQuant hot path on B200: encode -> score -> top-k.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one pass of the whole path over one batch of synthetic input:
tq_encode of every vector, then the estimates of the queries against all
codes and their top-10 (one tq_score_topk call when a workload has both,
which transforms and scores the queries once; else tq_topk alone).

Without --config every workload runs in one process -- tiny, kv, decode,
search, larged -- and ONE JSON line is printed.  Its headline (value,
ms_per_step, roofline, cpu_baseline, e2e) is large-d (10^6 x 3072 fp32 rows,
b = 4, 256 queries), the largest single-GPU workload; the others sit in its
"configs" object, each with its own timing, roofline and cpu_baseline.  The
headline times exactly --steps steps; every other workload repeats its step
until its timed region lasts at least a second (so the clock sampler sees it).
Inputs sit in HBM before a timed region; L2 (126 MB) is flushed by writing a
256 MB buffer between timed steps.

Multi-GPU: --gpus N > 1 starts N ranks itself (torchrun, one rank per GPU,
NCCL) unless it already runs under torchrun.  Every workload but search is
weak-scaled (each rank encodes and scores its own seeded batch; the vectors
are independent problems, so no data-path collective).  The search is
strong-scaled: one database of 10^6 rows sharded across the ranks, each
rank's top-10 made global and merged after one all-gather
(kv_cache_embedding_b200.sharded).  Times are the max over ranks.

--impl reference times the plain CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
import argparse
import json
import math
import os
import socket
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
HEADLINE = "larged"
ALL = ("tiny", "kv", "decode", "search", "larged")

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
                 desc="4096 x 128 fp32 rows (norms U[0.5,2]), 64 queries, b=4"),
    "search": dict(G=1, n=1_000_000, d=1536, b=4, x="unit", nq=1024, q="unit", k=10, score=False,
                   topk=True, desc="embedding search 1e6 x 1536 fp32 unit rows, 1024 queries, "
                                   "b=4, top-10"),
    "larged": dict(G=1, n=1_000_000, d=3072, b=4, x="rows", nq=256, q="gauss", k=10, score=True,
                   topk=True, desc="1e6 x 3072 fp32 rows (norms U[0.5,2]), 256 queries, "
                                   "b=4"),
}

FFMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # FP32 CUDA-core peak at max SM clock

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# a workload's dominant kernel, from one ncu capture (summaries under
# profiles/).  It is reported only while the kernel's sources still hash to
# what was captured.
NCU_TRAFFIC = {
    ("kv", "k_encode_tc"): {
        "sources": ["kv_cache_embedding_b200/csrc/tq_encode_tc.cu"],
        "sha1": "d0fba32e71c4e1608d47cd281935347fa9eba732",
        "bytes": 68254208 + 4477696,
    },
    # the encode call of the large-d workload: one 65,536-row chunk captured
    # (k_rownorm_split16, k_gemm_pair<1>, k_gemm_pair<2>: 7,318,083,584 bytes)
    # scaled by rows to 10^6, plus the once-per-call fp16 pieces of Pi and S
    # (k_split2h x 2: 77,417,984 bytes)
    ("larged", "encode"): {
        "sources": ["kv_cache_embedding_b200/csrc/tq_encode.cu",
                    "kv_cache_embedding_b200/csrc/tq_gemm_tc.cu",
                    "kv_cache_embedding_b200/csrc/tq_sm100.cuh",
                    "kv_cache_embedding_b200/csrc/tq_internal.cuh"],
        "sha1": "7eaf6b4b254e4974a13efe3b92089d613ff45741",
        "bytes": 111742511734,
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
def make_inputs(cfg, device, seed_offset=0, max_rows=None, rows=None):
    """(x [G, n, d], q [G, nq, d]) of a workload.  rows = (start, stop) keeps
    that slice of every group's rows (one shard of a database that is the same
    whatever the number of shards)."""
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
    if rows is not None:
        x = x[:, rows[0]:rows[1]].clone()
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


def launch_ranks(args):
    """Re-run this script as `--gpus` ranks under torchrun (rendezvous on
    127.0.0.1); returns torchrun's exit status."""
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


# ---------------------------------------------------------------- our arm
class Step:
    """One pass of the hot path with preallocated outputs and workspaces.
    With `shard` = (n_total, group) the top-k runs over a database sharded
    across ranks (local top-k, global ids, all-gather, merge)."""

    def __init__(self, tq, cfg, x, q, shard=None):
        import kv_cache_embedding_b200 as K
        self.K = K
        self.cfg = cfg
        self.tq = tq
        self.x, self.q = x, q
        self.shard = shard
        G, n, d, nq, k = cfg["G"], x.shape[1], cfg["d"], cfg["nq"], cfg["k"]
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
            if self.shard is not None:
                v, i = self.K.sharded.sharded_topk(tq, self.codes, self.q, self.cfg["k"],
                                                   self.shard[0], self.shard[1])
                self.topk[0].copy_(v)
                self.topk[1].copy_(i)
            else:
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


def alg_bytes_flops(cfg, n=None):
    G, d, b, nq, k = cfg["G"], cfg["d"], cfg["b"], cfg["nq"], cfg["k"]
    n = cfg["n"] if n is None else n
    esz = 2 if cfg["x"] == "kv" else 4
    rec = b * d // 8 + 8
    enc_bytes = G * n * (d * esz + rec)
    # two d x d products per vector (rotation, QJL projection); one for MSE-only
    enc_flops = (2.0 if cfg.get("variant", "prod") == "mse" else 4.0) * d * d * G * n
    score_bytes = G * n * rec + (G * nq * n * 4 if cfg["score"] else 0)
    score_flops = 4.0 * d * G * n * nq
    return dict(enc_bytes=enc_bytes, enc_flops=enc_flops, score_bytes=score_bytes,
                score_flops=score_flops, rec=rec, in_bytes=d * esz)


def encode_roofline(name, cfg, ab, enc_ms, pk, clocks):
    """Roofline of the encode call, the dominant kernel of every workload's
    step: achieved algorithmic FLOP/s (4 d^2 per vector, 2 d^2 for the
    MSE-only variant) against the peak of the unit it runs on.  The 16-bit
    tensor peak is the measured bf16 one (fp16 runs at the same rate): the
    burst figure, or the sustained one when the timed region ran under the
    power cap, divided by the mean number of 16-bit passes per product."""
    ach = ab["enc_flops"] / (enc_ms / 1e3) / 1e12
    mse = cfg.get("variant", "prod") == "mse"
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    bf16 = pk["bf16_sus"] if capped else pk["bf16"]
    which = "sustained" if capped else "burst"
    hbm = {"hbm_gbs": round(ab["enc_bytes"] / enc_ms / 1e6, 1),
           "hbm_frac": round(ab["enc_bytes"] / enc_ms / 1e6 / pk["hbm"], 4),
           "alg_bytes": ab["enc_bytes"]}
    if cfg["d"] == 128 and cfg["x"] == "kv" and not mse:
        peak = bf16 / 2.5
        return {"bound": "tensor", "achieved": round(ach, 2), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / peak, 4),
                "traffic": ncu_traffic(name, "k_encode_tc"),
                "kernel": "k_encode_tc (tq_encode: rotation (2 fp16 passes) + QJL (3) on "
                          "tcgen05, fused epilogue)",
                "peak_source": f"measured bf16 {which} (MEASURED_PEAKS.json) / 2.5 passes "
                               f"(fp16 = bf16 rate)" if pk["src"] == "measured" else
                               f"fallback bf16 {which} / 2.5 passes",
                "frac_of_3xtf32_fp32_equivalent": round(ach / (bf16 * 0.5 / 3.0), 4), **hbm}
    # tensor-core GEMMs on fp16 pieces: the rotation takes 3 passes for fp32
    # rows (2 x 2 pieces) and 2 for bf16 rows (one exact piece), the QJL 3
    p_rot = 2 if cfg["x"] == "kv" else 3
    passes = [p_rot] if mse else [p_rot, 3]
    peak = bf16 * len(passes) / sum(passes)
    if cfg["d"] % 256 == 0 and not mse:
        kernel = ("tq_encode call: k_gemm_pair<1> (rotation, bucketize in the epilogue) + "
                  "k_gemm_pair<2> (QJL, record packing in the epilogue) -- CTA-pair tcgen05 "
                  "GEMMs on fp16 pieces -- + k_rownorm_split16")
    else:
        kernel = ("tq_encode call: k_gemm_tc (rotation and QJL as tcgen05 GEMMs on fp16 "
                  "pieces) + k_rownorm_split16 + k_quantize16 + k_pack")
    return {"bound": "tensor", "achieved": round(ach, 2), "peak": round(peak, 1),
            "unit": "TFLOP/s", "frac": round(ach / peak, 4),
            "traffic": ncu_traffic(name, "encode") if cfg["n"] == CONFIGS[name]["n"] else None,
            "kernel": kernel,
            "peak_source": (f"measured bf16 {which} (MEASURED_PEAKS.json)" if pk["src"] == "measured"
                            else f"fallback bf16 {which}") +
                           f" / {sum(passes) / len(passes):g} passes (mean over the products)",
            **hbm}


def time_steps(run, flush, steps):
    """Device time (ms) of `steps` calls of run(), L2 flushed before each;
    one event pair per call on the current stream."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for a, b in ev:
        flush.zero_()
        a.record()
        run()
        b.record()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def graph_call_time(run, flush, reps=20, trials=5):
    """Device time (ms) of one call of run() inside a CUDA graph, L2 flushed
    before each call: a graph of `reps` x [flush, call] is timed with one
    event pair, a graph of `reps` x [flush] likewise, and the difference is
    divided by `reps` (median of `trials` replays each).  This leaves out the
    per-launch submission gaps of an eager stream and the event timer's
    granularity, which a single event pair around a ~50 us call does not."""
    def capture(fn):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fn()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                for _ in range(reps):
                    fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        return g

    def timed(g):
        ts = []
        for _ in range(trials):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    gf = capture(lambda: flush.zero_())
    gc = capture(lambda: (flush.zero_(), run()))
    ms = (timed(gc) - timed(gf)) / reps
    del gc, gf
    return ms


def e2e_time(tq, cfg, x, q, steps, dist, dev, shard):
    """End-to-end step through the public API with host buffers: every step
    copies its inputs from pinned host memory, runs the same calls and copies
    every result back to pinned host memory.  Two buffer sets and one stream
    per copy direction let the copies of neighbouring steps overlap the
    compute.  Returns (ms per step, h2d bytes, d2h bytes)."""
    xh = x.cpu().pin_memory()
    qh = q.cpu().pin_memory()
    bufs = []
    for _ in range(2):
        xd, qd = torch.empty_like(x), torch.empty_like(q)
        stp = Step(tq, cfg, xd, qd, shard)
        host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in stp.outputs()]
        bufs.append((xd, qd, stp, host))
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(m):
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

    run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    e0.record()
    run(steps)
    e1.record()
    torch.cuda.synchronize()
    ms = rank_max(dist, [e0.elapsed_time(e1) / steps], dev)[0]
    h2d = xh.numel() * xh.element_size() + qh.numel() * qh.element_size()
    d2h = sum(t.numel() * t.element_size() for t in bufs[0][3])
    return ms, h2d, d2h


def workload(name, args):
    """A workload's config, with its rows per group set by --rows (small cases
    of the same kernels for profiler captures)."""
    cfg = dict(CONFIGS[name])
    if getattr(args, "rows", None):
        cfg["n"] = int(args.rows)
        cfg["desc"] = cfg["desc"] + f" [rows per group set to {cfg['n']}]"
    return cfg


def bench_config(args, name, rank, world, dist, headline):
    """Time one workload; returns its JSON object (the headline's carries the
    top-level keys of the line)."""
    import kv_cache_embedding_b200 as K
    cfg = workload(name, args)
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    sharded = name == "search" and world > 1
    if sharded:  # one database across the ranks (strong scaling)
        span = K.sharded.shard_bounds(cfg["n"], world, rank)
        x, q = make_inputs(cfg, dev, rows=span)
        shard = (cfg["n"], None)
    else:
        x, q = make_inputs(cfg, dev, seed_offset=rank)
        shard = None
    tq = K.TurboQuant(cfg["d"], cfg["b"], seed=0, groups=cfg["G"], device=dev,
                      variant=cfg.get("variant", "prod"))
    step = Step(tq, cfg, x, q, shard)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    nlaunch, kernel_names = count_launches(step) if not args.no_count else (None, [])
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    # The step as one CUDA graph (the same public calls, captured once): its
    # replays are the timed steps.  Per-call times come from a second pass of
    # plain stream launches.  The sharded search (an NCCL all-gather in the
    # step) runs as plain launches.
    graph = None
    if not args.no_graph and not sharded:
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
    run = graph.replay if graph is not None else step.run
    # steps: exactly --steps for the headline; else enough for >= 1 s of timed region
    K_ = args.steps
    if not headline:
        est = statistics.median(time_steps(run, flush, 3))
        K_ = max(args.steps, min(20000, int(math.ceil(1000.0 / max(est, 1e-3)))))
        K_ = int(rank_max(dist, [K_], dev)[0])
    sampler = ClockSampler(dev)
    sampler.start()
    sampler.wait_first()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    tot_ms = sum(time_steps(run, flush, K_))
    if dist:
        dist.barrier()
    t1 = time.time()
    time.sleep(0.3)
    sampler.stop()
    # per-call breakdown, plain launches
    nb = min(K_, 50)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nb)]
    for i in range(nb):
        flush.zero_()
        step.run(evs[i])
    torch.cuda.synchronize()
    enc = sum(e[0].elapsed_time(e[1]) for e in evs) / nb
    sco = sum(e[1].elapsed_time(e[2]) for e in evs) / nb
    tpk = sum(e[2].elapsed_time(e[3]) for e in evs) / nb
    tot_ms, enc, sco, tpk = rank_max(dist, [tot_ms, enc, sco, tpk], dev)
    ms_step = tot_ms / K_
    n_rank = x.shape[1]
    units = cfg["G"] * cfg["n"] if sharded else cfg["G"] * n_rank * world
    value = units * K_ / (tot_ms / 1e3) / 1e6

    e2e_steps = max(2, min(args.steps, 5 if cfg["d"] >= 256 else 20))
    e2e_ms, h2d, d2h = e2e_time(tq, cfg, x, q, e2e_steps, dist, dev, shard)

    ab = alg_bytes_flops(cfg, n_rank)
    pk = peaks()
    out = {
        "metric": METRIC, "value": round(value, 4), "unit": "Mvec/s", "n_gpus": world,
        "steps": K_, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "strong" if sharded else "weak",
        "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; shapes of the pages' KV-cache / embedding workloads)",
        "config": {"workload": f"{name}: {cfg['desc']}", "G": cfg["G"], "n": cfg["n"],
                   "d": cfg["d"], "b": cfg["b"], "queries_per_group": cfg["nq"], "k": cfg["k"],
                   "l2": "flushed (256 MB write) between timed steps",
                   "launch": "CUDA graph of the step" if graph is not None else "stream launches",
                   "parallelism": (f"sharded database over {world} ranks (local top-k, all-gather, "
                                   f"merge)") if sharded else
                   f"dp{world} (independent batches per GPU)"},
        "encode": {"ms": round(enc, 5), "mvec_s": round(cfg["G"] * n_rank / enc / 1e3, 3),
                   "gbs": round(ab["enc_bytes"] / enc / 1e6, 2),
                   "hbm_frac": round(ab["enc_bytes"] / enc / 1e6 / pk["hbm"], 4)},
        "roofline": None,
        "e2e": {"value": round(units / e2e_ms / 1e3, 4), "unit": "Mvec/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": (nlaunch * K_) if nlaunch is not None else None,
        "gpu_launches_per_step": nlaunch,
        "kernels": kernel_names,
        "clocks": sampler.summary(t0, t1),
        "peaks": pk,
        "compression": {"record_bytes": ab["rec"], "input_bytes": ab["in_bytes"],
                        "vs_input": round(ab["in_bytes"] / ab["rec"], 3),
                        "vs_fp32": round(cfg["d"] * 4 / ab["rec"], 3)},
    }
    out["roofline"] = encode_roofline(name, cfg, ab, enc, pk, out["clocks"])
    if step.combined:
        # tq_score_topk: the score matrix and the top-k lists from one scoring pass
        sg = ab["score_bytes"] / sco / 1e6
        out["score_topk"] = {"ms": round(sco, 5),
                             "scores_s": round(cfg["G"] * cfg["nq"] * n_rank / sco * 1e3, 1),
                             "gbs": round(sg, 2), "hbm_frac": round(sg / pk["hbm"], 4),
                             "call": "tq_score_topk (scores written + top-k of the same pass)"}
    elif cfg["topk"]:
        out["topk"] = {"ms": round(tpk, 5),
                       "scores_s": round(cfg["G"] * cfg["nq"] * n_rank / tpk * 1e3, 1),
                       "call": "tq_topk" + (" per shard + all-gather + tq_topk_merge"
                                            if sharded else "")}
    if name in ("kv", "decode") and rank == 0:
        out["score_alone"] = score_alone_time(tq, cfg, step, flush, args, nq=cfg["nq"])
    if name == "decode" and rank == 0:
        out["score_1q_per_kv_head"] = score_alone_time(tq, cfg, step, flush, args, nq=1)
        out["fp32_baseline"] = fp32_baseline(cfg, x, q, flush, args)
        out["attention"] = attention_decode_time(cfg, x, q, flush, args)
    if name == "search":
        out["recall_at_10"] = search_recall(tq, step, x, q, cfg, shard)
    del graph, step
    return out


def score_alone_time(tq, cfg, step, flush, args, nq):
    """tq_score alone (query transform + scoring of nq queries per group over
    the step's codes), L2 flushed before each call; bytes = the records read
    and the scores written."""
    q = step.q[:, :nq].contiguous()
    out = torch.empty(cfg["G"], nq, step.codes.n, dtype=torch.float32, device=q.device)
    for _ in range(3):
        tq.score(step.codes, q, out=out)
    ts = time_steps(lambda: tq.score(step.codes, q, out=out), flush, max(10, min(args.steps, 50)))
    ms = statistics.median(ts)
    gms = graph_call_time(lambda: tq.score(step.codes, q, out=out), flush)
    rec = cfg["b"] * cfg["d"] // 8 + 8
    byts = cfg["G"] * step.codes.n * rec + out.numel() * 4
    pk = peaks()
    return {"ms": round(ms, 5), "queries_per_group": nq, "gbs": round(byts / ms / 1e6, 1),
            "hbm_frac": round(byts / ms / 1e6 / pk["hbm"], 4),
            "scores_s": round(out.numel() / ms * 1e3, 1), "call": "tq_score",
            "graph_ms": round(gms, 5), "graph_gbs": round(byts / gms / 1e6, 1),
            "timing": "ms: event pair around each eager call; graph_ms: per call inside a CUDA graph"}


def search_recall(tq, step, x, q, cfg, shard):
    """recall@10 of the step's top-10 (estimates from 4-bit codes) against the
    exact fp32 top-10 of the same database (tq_exact_topk), over every query;
    sharded databases merge the exact lists like the estimated ones."""
    import kv_cache_embedding_b200 as K
    k = cfg["k"]
    step.run()
    est = step.topk[1]
    if shard is not None:
        _, ex = K.sharded.sharded_topk(None, x, q, k, shard[0], shard[1],
                                       local_topk=lambda xs, qq, kk: K.exact_topk(xs, qq, kk))
    else:
        _, ex = K.exact_topk(x, q, k)
    torch.cuda.synchronize()
    e = est.reshape(-1, k).cpu()
    t = ex.reshape(-1, k).cpu()
    hits = sum(len(set(a.tolist()) & set(b.tolist())) for a, b in zip(e, t))
    return {"value": round(hits / (k * e.shape[0]), 5), "queries": int(e.shape[0]),
            "truth": "tq_exact_topk (fp32 inner products of the unquantized rows)"}


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
    ts = time_steps(lambda: tk.attention_decode(kc, tv, vc, q, out=out), flush,
                    max(3, min(args.steps, 50)))
    ms = sum(ts) / len(ts)
    gms = graph_call_time(lambda: tk.attention_decode(kc, tv, vc, q, out=out), flush)
    byts = (kc.codes.numel() * 4 + kc.xnorm.numel() * 8 + vc.codes.numel() * 4 +
            vc.xnorm.numel() * 4 + q.numel() * q.element_size() + out.numel() * 4)
    return {"ms": round(ms, 5), "gbs": round(byts / ms / 1e6, 1), "graph_ms": round(gms, 5),
            "values": "4-bit MSE-only records (seeded keys-like rows)", "scale": "1/sqrt(d)"}


def fp32_baseline(cfg, x, q, flush, args):
    """Unquantized fp32 keys: logits kernel time vs tq_score on packed codes."""
    import kv_cache_embedding_b200 as K
    keys = x.float()
    out = torch.empty(cfg["G"], cfg["nq"], cfg["n"], dtype=torch.float32, device=x.device)
    for _ in range(3):
        K.logits_fp32(keys, q, out)
    ts = time_steps(lambda: K.logits_fp32(keys, q, out), flush, max(3, min(args.steps, 50)))
    ms = sum(ts) / len(ts)
    gms = graph_call_time(lambda: K.logits_fp32(keys, q, out), flush)
    byts = keys.numel() * 4 + out.numel() * 4
    return {"ms": round(ms, 5), "gbs": round(byts / ms / 1e6, 1), "graph_ms": round(gms, 5)}


# ---------------------------------------------------------------- oracle arm
def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def omp_threads(n):
    """Set the OpenMP thread count of the oracle library (libgomp); returns
    False when that runtime cannot be reached."""
    import ctypes
    try:
        ctypes.CDLL("libgomp.so.1").omp_set_num_threads(int(n))
        return True
    except OSError:
        return False


class OracleSample:
    """The oracle's encode -> score -> top-k on a bounded sample of a
    workload: the first rows of group 0, with one group's parameters built
    once (outside the timing)."""

    def __init__(self, cfg):
        from oracle import oracle as O
        self.O = O
        self.cfg = cfg
        x, q = make_inputs(cfg, "cpu", max_rows=65536)
        self.x = x[0].to(torch.float64).numpy()
        self.q = q[0].to(torch.float64).numpy()
        self.mse = cfg.get("variant", "prod") == "mse"
        d, b = cfg["d"], cfg["b"]
        self.params = O.MseParams(d, b, 0) if self.mse else O.Params(d, b, 0)

    def run(self, rows):
        O, P = self.O, self.params
        xs = self.x[:rows]
        t = time.perf_counter()
        if self.mse:
            codes, xn, rn = O.mse_encode(P, xs)
            s = O.mse_score(P, codes, xn, self.q)
        else:
            codes, xn, rn = O.encode(P, xs)
            s = O.score(P, codes, xn, rn, self.q)
        O.topk(s, min(self.cfg["k"], rows))
        return time.perf_counter() - t

    def sized(self, target_s):
        """(rows, seconds) of a sample grown by 4x until it takes target_s / 4."""
        n = self.x.shape[0]
        rows = min(n, 256)
        dt = self.run(rows)
        while dt < target_s / 4 and rows < n:
            rows = min(n, rows * 4)
            dt = self.run(rows)
        return rows, dt

    def describe(self, rows):
        c = self.cfg
        return (f"{rows} of the {c['G'] * c['n']} vectors (group 0), oracle encode + score of "
                f"{c['nq']} queries + top-{c['k']}, extrapolated per vector")

    def flagged_rate(self, rows=None):
        """Fraction of coordinates whose fp64 rotated value lies within 1e-5 sigma
        of a Lloyd-Max boundary (the codes the parity rules exempt)."""
        import numpy as np
        rows = rows or (2048 if self.cfg["d"] <= 128 else 256)
        if self.mse:
            _, _, _, y, _ = self.O.mse_encode(self.params, self.x[:rows], diagnostics=True)
        else:
            _, _, _, y, _, _ = self.O.encode(self.params, self.x[:rows], diagnostics=True)
        beta = np.asarray(self.params.beta, dtype=np.float64)
        if beta.size == 0:
            return {"value": 0.0, "coordinates": int(y.size)}
        band = 1e-5 / math.sqrt(self.cfg["d"])
        near = np.zeros(y.shape, dtype=bool)
        for bj in beta:
            near |= np.abs(y - bj) < band
        return {"value": float(near.mean()), "coordinates": int(y.size),
                "band": "1e-5 sigma, sigma = 1/sqrt(d)", "rows": int(y.shape[0])}


def cpu_baseline(cfg, target_s):
    """The oracle timed on the host cores (all of them, then one), for a
    workload's line."""
    o = OracleSample(cfg)
    rows, dt = o.sized(target_s)
    cores = int(os.environ.get("OMP_NUM_THREADS", cpu_cores()))
    out = {"value": rows / dt / 1e6, "unit": "Mvec/s", "cores": cores, "kind": "oracle",
           "sample": o.describe(rows), "cpu_model": cpu_model()}
    if omp_threads(1):
        r1 = max(16, rows // 16)
        t1 = o.run(r1)
        omp_threads(cores)
        out["one_core"] = {"value": r1 / t1 / 1e6, "unit": "Mvec/s",
                           "sample": f"{r1} vectors, OpenMP limited to 1 thread"}
    out["flagged_coordinate_rate"] = o.flagged_rate()
    return out


def run_reference(args, cfg, name):
    o = OracleSample(cfg)
    rows, _ = o.sized(max(0.5, 60.0 / max(args.steps + args.warmup, 1)))
    times = []
    for i in range(args.warmup + args.steps):
        dt = o.run(rows)
        if i >= args.warmup:
            times.append(dt)
    secs = sum(times)
    value = rows * len(times) / secs / 1e6
    cores = int(os.environ.get("OMP_NUM_THREADS", cpu_cores()))
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mvec/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / len(times) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{name}: {cfg['desc']}", "G": cfg["G"], "n": cfg["n"],
                   "d": cfg["d"], "b": cfg["b"]},
        "cpu_baseline": {"value": value, "unit": "Mvec/s", "cores": cores, "kind": "oracle",
                         "sample": o.describe(rows), "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "Mvec/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=None, choices=sorted(CONFIGS),
                    help="one workload only (default: all of them, large-d as the headline)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time plain stream launches instead of replays of the step's CUDA graph")
    ap.add_argument("--no-count", action="store_true",
                    help="skip the profiler-based launch count (for runs under ncu)")
    ap.add_argument("--rows", type=int, default=None,
                    help="rows per group instead of the workload's (small cases for ncu)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_ranks(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    names = (args.config,) if args.config else ALL
    head = args.config or HEADLINE
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, workload(head, args), head)))
        return 0

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as td
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = td
    results = {}
    for name in names:
        results[name] = bench_config(args, name, rank, world, dist, headline=(name == head))
        torch.cuda.empty_cache()
    out = results[head]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        for name in names:
            results[name]["cpu_baseline"] = cpu_baseline(workload(name, args),
                                                         10.0 if name == head else 4.0)
    if len(names) > 1:
        out["configs"] = {nm: {k: v for k, v in r.items()
                               if k not in ("metric", "higher_is_better", "vs_baseline", "data",
                                            "peaks", "unit", "n_gpus", "warmup")}
                          for nm, r in results.items() if nm != head}
    if rank == 0:
        print(json.dumps(out))
    if dist:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
