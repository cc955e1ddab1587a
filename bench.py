#!/usr/bin/env python
"""Benchmark of the TurboQuant codec on B200.

Default workload: one Llama-3.1-8B-shaped attention layer - 8 KV heads x
32768 tokens, d = 128, 32 query heads (GQA 4), bf16 K/V from the synthetic
law (per-channel lognormal(0, 0.5) scales, 4 outlier channels x20, per-token
lognormal(0, 0.3) norms).  One step = the whole hot path at b = 3 and b = 4:
    tq_quantize(K, product code), tq_quantize(V, MSE code),
    tq_logits(32 decode queries over the 262144 compressed keys).
Metric: compressed-key logits, keys/s (keys scored per second over the whole
step, both bit widths), with per-kernel HBM GB/s and fractions of 8 TB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload layer|decode|quantize|search|polar|project]

N > 1 runs under torchrun, one rank per GPU, each rank a full independent
layer (weak scaling, no collective on the data path).  Rank 0 prints one JSON
line.  --impl reference times the CPU oracle (fp64 numpy) on a bounded
sample of the same workload on the host cores.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HBM_NOMINAL_GBS = 8000.0
METRIC = "compressed-key logits keys/s and HBM GB/s (frac of 8 TB/s) at b=3,4"
VALUE_DEF = ("keys per second through the whole step (tq_quantize of K and V, tq_logits of the 32 decode "
             "queries), b=3 and b=4; tq_logits alone, with GB/s and fractions of 8 TB/s, under 'logits'")
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="layer",
                    choices=["layer", "decode", "quantize", "search", "polar", "project"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-kernels", action="store_true")
    ap.add_argument("--decode-batch", type=int, default=64, help="sequences of the decode workload (64)")
    ap.add_argument("--no-configs", action="store_true")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_bf16_peak():
    """Dense bf16 FLOP/s of this machine's B200s (sustained, for a kernel timed in a loop)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        for k in ("bf16_tflops_sustained", "bf16_tflops"):
            if k in d:
                return float(d[k]) * 1e12
    return 1.4e15


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/throttle sampling around the timed region: sampling runs
    every 20 ms from before the warm-up (start() waits for the first sample) to
    after the timing; stop() keeps the samples within 150 ms of the timed window
    (set by window()), or the nearest sample on each side if none falls inside."""
    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = str(gpu_index)
        try:
            import torch
            u = str(torch.cuda.get_device_properties(gpu_index).uuid)
            self.idx = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            pass
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            deadline = time.time() + 5.0
            while time.time() < deadline and os.path.getsize(self.path) == 0:
                time.sleep(0.02)
        except Exception:
            self.proc = None

    def window(self, t0, t1):
        self.t0, self.t1 = t0, t1

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                rows.append(dict(t=ts, sm=float(parts[1]), smax=float(parts[2]), hw=parts[5], hwt=parts[6],
                                 swt=parts[7], swp=parts[8]))
            except (ValueError, IndexError):
                continue
        os.unlink(self.path)
        if not rows:
            return None
        if self.t0 is not None:
            inside = [r for r in rows if self.t0 - 0.15 <= r["t"] <= self.t1 + 0.15]
            if not inside:
                before = [r for r in rows if r["t"] < self.t0]
                after = [r for r in rows if r["t"] > self.t1]
                inside = before[-1:] + after[:1]
            rows = inside or rows
        reasons = set()
        for r in rows:
            for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                            ("swp", "sw_power_cap")):
                if r[k].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# --------------------------------------------------------------------------- distributed
def dist_setup(args=None):
    """One process per GPU (RANK/LOCAL_RANK/WORLD_SIZE/MASTER_* from the launcher).
    NCCL on GPUs; gloo where there is no GPU (the host-side plumbing, tested on CPU)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def allmax(world, v):
    """Maximum of v over the ranks (every rank takes part, in the same order)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world, units_per_rank, max_ms):
    """Whole-job throughput: every rank processes units_per_rank; the job takes
    the slowest rank's time."""
    return world * units_per_rank / (max_ms / 1e3)


# --------------------------------------------------------------------------- workloads
class Layer:
    """One attention layer: 8 KV heads x 32768 tokens, 32 query heads, b = 3 and 4."""
    H_KV, T, D, GROUP = 8, 32768, 128, 4
    BITS = (3, 4)

    def __init__(self, tq, wl, torch):
        self.tq, self.torch = tq, torch
        n = self.H_KV * self.T
        self.n = n
        K = wl.kv_block(1, self.H_KV, self.T, self.D, seed=wl.SEED_KEYS).reshape(n, self.D)
        V = wl.kv_block(1, self.H_KV, self.T, self.D, seed=wl.SEED_VALUES).reshape(n, self.D)
        q = wl.queries(self.H_KV * self.GROUP, self.D, seed=wl.SEED_QUERIES)
        self.K = torch.from_numpy(K).to(torch.bfloat16).cuda()
        self.V = torch.from_numpy(V).to(torch.bfloat16).cuda()
        self.q = torch.from_numpy(q).cuda()
        self.kp, self.vp, self.bufs = {}, {}, {}
        for b in self.BITS:
            kp = tq.Params(self.D, b, tq.TQ_MODE_PROD, 128, wl.SEED_PARAMS)
            vp = tq.Params(self.D, b, tq.TQ_MODE_MSE, 0, wl.SEED_PARAMS + 1)
            self.kp[b], self.vp[b] = kp, vp
            dev = "cuda"
            self.bufs[b] = dict(
                kc=torch.empty(kp.code_bytes(n), dtype=torch.uint8, device=dev),
                kn=torch.empty(n, dtype=torch.int16, device=dev),
                krn=torch.empty(n, dtype=torch.int16, device=dev),
                vc=torch.empty(vp.code_bytes(n), dtype=torch.uint8, device=dev),
                vn=torch.empty(n, dtype=torch.int16, device=dev),
                lg=torch.empty((self.q.shape[0], self.T), dtype=torch.float32, device=dev),
                ws=torch.empty(tq.tq_logits_workspace(kp, self.q.shape[0]), dtype=torch.uint8, device=dev))
        self.launches_per_step = len(self.BITS) * 4   # quantize K, quantize V, logits prep + scan

    def calls(self, inputs=None):
        """The step as a list of (label, callable); `inputs` = (K, V, q) device tensors (default: the layer's)."""
        tq = self.tq
        K, V, q = inputs if inputs is not None else (self.K, self.V, self.q)
        out = []
        for b in self.BITS:
            B = self.bufs[b]
            kp, vp = self.kp[b], self.vp[b]
            out.append((f"tq_quantize_K_b{b}", lambda kp=kp, B=B: tq.tq_quantize(kp, K, B["kc"], B["kn"], B["krn"])))
            out.append((f"tq_quantize_V_b{b}", lambda vp=vp, B=B: tq.tq_quantize(vp, V, B["vc"], B["vn"])))
            out.append((f"tq_logits_b{b}", lambda kp=kp, B=B: tq.tq_logits(kp, q, self.GROUP, B["kc"], B["kn"],
                                                                           B["krn"], self.T, self.H_KV, B["lg"],
                                                                           B["ws"])))
        return out

    def keys_per_step(self):
        return len(self.BITS) * self.n

    def bytes_of(self, label):
        """Algorithmic bytes one call must move (inputs read + outputs written)."""
        b = int(label[-1])
        n, d = self.n, self.D
        kc = self.kp[b].code_bytes(n)
        if label.startswith("tq_quantize_K"):
            return n * d * 2 + kc + 4 * n
        if label.startswith("tq_quantize_V"):
            return n * d * 2 + self.vp[b].code_bytes(n) + 2 * n
        nq = self.q.shape[0]
        return kc + 4 * n + nq * d * 4 + nq * self.T * 4

    def metric_bytes(self, b):
        """Bytes the logits metric counts: packed codes + norms + residual norms + queries."""
        return self.kp[b].code_bytes(self.n) + 4 * self.n + self.q.numel() * 4

    def host_inputs(self):
        return [self.K, self.V, self.q]

    def host_outputs(self):
        return [self.bufs[b]["lg"] for b in self.BITS]


# --------------------------------------------------------------------------- timing helpers
def l2_flush(torch, buf):
    buf.zero_()


def time_steps(torch, wk, steps, warmup, world, flush, sampler=None):
    """Device-timed steps: per-step and per-call CUDA events on the launching stream."""
    calls = wk.calls()
    for _ in range(warmup):
        for _, f in calls:
            f()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(steps)]
    t_wall0 = time.time()
    for s in range(steps):
        l2_flush(torch, flush)
        ev[s][0].record()
        for i, (_, f) in enumerate(calls):
            f()
            ev[s][i + 1].record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    if sampler is not None:
        sampler.window(t_wall0, t_wall1)
    step_ms = [ev[s][0].elapsed_time(ev[s][-1]) for s in range(steps)]
    per_call = {}
    for i, (label, _) in enumerate(calls):
        per_call[label] = [ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps)]
    return step_ms, per_call


def time_e2e(torch, wk, steps, warmup):
    """Same step through the public API with pinned host buffers: every step copies
    its inputs host -> device and reads its logits back device -> host, all inside
    the timed region.  The next step's inputs are uploaded on a second stream into
    the other of two device input sets while the current step computes (events
    order each copy before its step and after the step that last read that set)."""
    hin = [t.cpu().pin_memory() for t in wk.host_inputs()]
    hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in wk.host_outputs()]
    dsets = [wk.host_inputs(), [torch.empty_like(t) for t in wk.host_inputs()]]
    dout = wk.host_outputs()
    calls = [wk.calls(tuple(ds)) for ds in dsets]
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]

    def upload(k):
        with torch.cuda.stream(copy):
            for h, d in zip(hin, dsets[k]):
                d.copy_(h, non_blocking=True)
            copied[k].record(copy)

    def run(n):
        upload(0)
        for s in range(n):
            k = s % 2
            if s + 1 < n:
                if s >= 1:
                    copy.wait_event(consumed[1 - k])   # step s-1 has finished reading that set
                upload(1 - k)
            comp.wait_event(copied[k])
            for _, f in calls[k]:
                f()
            consumed[k].record(comp)
            for h, d in zip(hout, dout):
                h.copy_(d, non_blocking=True)

    run(warmup)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    copy.wait_event(e0)
    run(steps)
    e1.record(comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = sum(t.numel() * t.element_size() for t in hout)
    return ms, h2d, d2h


def logits_isolated(torch, tq, wk, reps_min=8):
    """tq_logits alone on L2-cold inputs: rotate over copies of the codes totalling > 4x L2,
    launches captured in a CUDA graph; returns {bits: (us per call, metric bytes)}."""
    res = {}
    for b in wk.BITS:
        B = wk.bufs[b]
        per_copy = B["kc"].numel() + 2 * B["kn"].numel() * 2
        ncopy = max(reps_min, int(4 * L2_BYTES // per_copy) + 1)
        copies = [(B["kc"].clone(), B["kn"].clone(), B["krn"].clone()) for _ in range(ncopy)]
        kp = wk.kp[b]

        def run_all():
            for kc, kn, krn in copies:
                tq.tq_logits(kp, wk.q, wk.GROUP, kc, kn, krn, wk.T, wk.H_KV, B["lg"], B["ws"])

        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            run_all()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                run_all()
        torch.cuda.current_stream().wait_stream(s)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1000.0 / (reps * ncopy)
        # single-call latency (stream launch, L2-cold copy)
        e0.record()
        tq.tq_logits(kp, wk.q, wk.GROUP, copies[0][0], copies[0][1], copies[0][2], wk.T, wk.H_KV, B["lg"], B["ws"])
        e1.record()
        torch.cuda.synchronize()
        lat = e0.elapsed_time(e1) * 1000.0
        res[b] = (us, wk.metric_bytes(b), lat)
        del copies, g
        torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------------------- CPU oracle
def cpu_oracle_layer(sample_tokens=16384):
    """The oracle (fp64 numpy, as it stands) on a bounded sample of the layer workload:
    all 8 heads x `sample_tokens` tokens, b = 3 and 4, quantize K and V + logits."""
    import workloads as wl
    from oracle import codec, estimate
    from oracle.codebook import stored_codebook
    from oracle.params import sign_flips, qjl_matrix
    H, T, d, group = Layer.H_KV, sample_tokens, Layer.D, Layer.GROUP
    K = wl.kv_block(1, H, T, d, seed=wl.SEED_KEYS).reshape(-1, d)
    V = wl.kv_block(1, H, T, d, seed=wl.SEED_VALUES).reshape(-1, d)
    q = wl.queries(H * group, d, seed=wl.SEED_QUERIES)
    t0 = time.perf_counter()
    for b in Layer.BITS:
        c, t = stored_codebook(128, b - 1)
        cv, tv = stored_codebook(128, b)
        Dk, S = sign_flips(wl.SEED_PARAMS, 128), qjl_matrix(wl.SEED_PARAMS, 128, 128)
        Dv = sign_flips(wl.SEED_PARAMS + 1, 128)
        ke = codec.encode(K, Dk, c, t, S)
        kbuf = codec.pack(ke["idx"], ke["signs"], b - 1, 128)
        ve = codec.encode(V, Dv, cv, tv)
        codec.pack(ve["idx"], None, b, 0)
        idx, sg = codec.unpack(kbuf, K.shape[0], 128, b - 1, 128)
        estimate.logits_gqa(q, Dk, S, idx, sg, ke["norm_f16"], ke["rnorm_f16"], c, 128, H, group, T)
    dt = time.perf_counter() - t0
    keys = len(Layer.BITS) * H * T
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    return keys / dt, cores, dt, f"8 heads x {T} tokens (of 32768), b=3 and b=4: quantize K and V + logits"


def cpu_oracle_one_core():
    """The oracle on one host core (BLAS limited to one thread): config 0 whole (4096 fp32 keys,
    16 queries, b = 4: quantize + logits) and a 16384-vector sample of config 3 (bf16, product
    code at b = 2, 3, 4)."""
    import workloads as wl
    from oracle import codec, estimate
    from oracle.codebook import stored_codebook
    from oracle.params import sign_flips, qjl_matrix
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        return None
    with threadpool_limits(limits=1):
        Dk, S = sign_flips(wl.SEED_PARAMS, 128), qjl_matrix(wl.SEED_PARAMS, 128, 128)
        x = wl.head_vectors(4096, 128, seed=wl.SEED_KEYS, token_scale=False)
        q = wl.queries(16, 128)
        c, t = stored_codebook(128, 3)
        t0 = time.perf_counter()
        e = codec.encode(x, Dk, c, t, S)
        buf = codec.pack(e["idx"], e["signs"], 3, 128)
        idx, sg = codec.unpack(buf, 4096, 128, 3, 128)
        estimate.logits_gqa(q, Dk, S, idx, sg, e["norm_f16"], e["rnorm_f16"], c, 128, 1, 16, 4096)
        cfg0 = time.perf_counter() - t0
        n3 = 16384
        x3 = wl.to_bf16(wl.head_vectors(n3, 128, seed=wl.SEED_KEYS))
        per = {}
        for b in (2, 3, 4):
            c, t = stored_codebook(128, b - 1)
            t0 = time.perf_counter()
            e = codec.encode(x3, Dk, c, t, S)
            codec.pack(e["idx"], e["signs"], b - 1, 128)
            per[f"b{b}"] = n3 / (time.perf_counter() - t0)
    return {"cores": 1, "config0_seconds": round(cfg0, 3),
            "config0": "4096 fp32 keys x 16 queries, b=4: quantize + logits",
            "config3_vectors_per_s": {k: round(v, 1) for k, v in per.items()},
            "config3_sample": f"{n3} of 2^20 bf16 vectors, product code m=128"}


# --------------------------------------------------------------------------- traffic record
def traffic_record(kernel_file_label):
    """ncu-derived DRAM bytes per launch from profiles/traffic.json, or None if the
    kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel_file_label)
    if not rec:
        return None
    src = os.path.join(ROOT, "vector_quantization_randomized_b200", "csrc", rec["source"])
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return rec["bytes_per_launch"] if h == rec["source_sha"] else None


# --------------------------------------------------------------------------- secondary workloads
def gpu_kv(torch, n_seq, n_heads, n_tokens, d, seed):
    """Keys/values with the synthetic law, drawn on the GPU (bf16 [n_seq*n_heads*n_tokens, d]).
    Same law as workloads.head_vectors; used where host generation of GBs would dominate."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    out = torch.empty((n_seq * n_heads, n_tokens, d), dtype=torch.bfloat16, device="cuda")
    for i in range(n_seq * n_heads):
        sigma = torch.exp(0.5 * torch.randn(d, generator=g, device="cuda"))
        outl = torch.randperm(d, generator=g, device="cuda")[:4]
        sigma[outl] *= 20.0
        rho = torch.exp(0.3 * torch.randn(n_tokens, generator=g, device="cuda"))
        z = torch.randn((n_tokens, d), generator=g, device="cuda")
        out[i] = (z * sigma[None, :] * rho[:, None]).to(torch.bfloat16)
    return out.reshape(-1, d)


def measure_decode(torch, tq, wl, steps, warmup, peak, sparse=True, batch=64):
    """Decode attention, `batch` (64) sequences x 8 KV heads x 16384 tokens, d 128, 32 query heads:
    K product code b = 3, V MSE code b = 3 (inputs drawn on the GPU, then quantized)."""
    ev = lambda: torch.cuda.Event(enable_timing=True)
    B, Hkv, T, d, Hq = batch, 8, 16384, 128, 32
    kp = tq.Params(d, 3, tq.TQ_MODE_PROD, 128, wl.SEED_PARAMS)
    vp = tq.Params(d, 3, tq.TQ_MODE_MSE, 0, wl.SEED_PARAMS + 1)
    n = B * Hkv * T
    bufs = {}
    for name, p, seed in (("k", kp, wl.SEED_KEYS), ("v", vp, wl.SEED_VALUES)):
        x = gpu_kv(torch, B, Hkv, T, d, seed)
        c = torch.empty(p.code_bytes(n), dtype=torch.uint8, device="cuda")
        nn = torch.empty(n, dtype=torch.int16, device="cuda")
        rn = torch.empty(n, dtype=torch.int16, device="cuda") if p.mode == tq.TQ_MODE_PROD else None
        tq.tq_quantize(p, x, c, nn, rn)
        torch.cuda.synchronize()
        del x
        bufs[name] = (c, nn, rn)
    q = torch.randn((B, Hq, d), device="cuda")
    out = torch.empty((B, Hq, d), device="cuda")
    ws = torch.empty(tq.tq_decode_attn_workspace(kp, B, Hq, Hkv, T), dtype=torch.uint8, device="cuda")
    sl = torch.full((B,), T, dtype=torch.int32, device="cuda")

    def timed(run):
        for _ in range(warmup):
            run()
        torch.cuda.synchronize()
        e0, e1 = ev(), ev()
        e0.record()
        for _ in range(steps):
            run()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    ms = timed(lambda: tq.tq_decode_attn(kp, vp, q, Hkv, bufs["k"][0], bufs["k"][1], bufs["k"][2], bufs["v"][0],
                                         bufs["v"][1], sl, T, out, ws))
    mbytes = bufs["k"][0].numel() + 4 * n + bufs["v"][0].numel() + 2 * n + q.numel() * 4
    gbs = mbytes / (ms / 1e3) / 1e9
    res = {"us": round(ms * 1000, 2), "tokens_per_s": n / (ms / 1e3), "metric_bytes": mbytes, "gbs": round(gbs, 1),
           "frac_8tbs": round(gbs / HBM_NOMINAL_GBS, 4), "frac_measured": round(gbs / peak, 4),
           "workload": f"decode-{B}x8x16384-Kprod3-Vmse3-hq32", "inputs": f"> L2 ({mbytes / 1e6:.0f} MB of codes)"}
    # the same values in the token-sliced layout: the tensor-memory decode
    vps = tq.Params(d, 3, tq.TQ_MODE_MSE, 0, wl.SEED_PARAMS + 1, layout=tq.TQ_LAYOUT_SLICED)
    x = gpu_kv(torch, B, Hkv, T, d, wl.SEED_VALUES)
    vcs = torch.empty(vps.code_bytes(n), dtype=torch.uint8, device="cuda")
    vns = torch.empty(n, dtype=torch.int16, device="cuda")
    tq.tq_quantize(vps, x, vcs, vns)
    torch.cuda.synchronize()
    del x
    ms_t = timed(lambda: tq.tq_decode_attn(kp, vps, q, Hkv, bufs["k"][0], bufs["k"][1], bufs["k"][2], vcs, vns, sl, T,
                                           out, ws))
    gbs_t = mbytes / (ms_t / 1e3) / 1e9
    res["tensor_memory"] = {"us": round(ms_t * 1000, 2), "tokens_per_s": n / (ms_t / 1e3), "gbs": round(gbs_t, 1),
                            "frac_measured": round(gbs_t / peak, 4),
                            "how": "values in the token-sliced layout (tq_params.layout = 1): decode_tc_kernel"}
    del vcs, vns
    if sparse:
        sp = {}
        for eps in (1e-4, 1e-3):
            ms_s = timed(lambda: tq.tq_decode_attn_sparse(kp, vp, q, Hkv, bufs["k"][0], bufs["k"][1], bufs["k"][2],
                                                          bufs["v"][0], bufs["v"][1], sl, T, out, ws, v_eps=eps))
            sp[f"v_eps={eps:g}"] = {"us": round(ms_s * 1000, 2), "tokens_per_s": n / (ms_s / 1e3)}
        res["sparse_v"] = sp
    del bufs, ws
    torch.cuda.empty_cache()
    return res


def measure_quantize(torch, tq, wl, steps, warmup, peak):
    """tq_quantize on 2^20 bf16 vectors, d 128, product code m = 128, at b = 2, 3, 4
    (268 MB of input per call: larger than L2)."""
    ev = lambda: torch.cuda.Event(enable_timing=True)
    n, d = 1 << 20, 128
    x = gpu_kv(torch, 1, 8, n // 8, d, wl.SEED_KEYS)
    res = {}
    for b in (2, 3, 4):
        p = tq.Params(d, b, tq.TQ_MODE_PROD, 128, wl.SEED_PARAMS)
        c = torch.empty(p.code_bytes(n), dtype=torch.uint8, device="cuda")
        nn = torch.empty(n, dtype=torch.int16, device="cuda")
        rn = torch.empty(n, dtype=torch.int16, device="cuda")
        run = lambda: tq.tq_quantize(p, x, c, nn, rn)
        for _ in range(warmup):
            run()
        torch.cuda.synchronize()
        e0, e1 = ev(), ev()
        e0.record()
        for _ in range(steps):
            run()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        byts = n * d * 2 + c.numel() + 4 * n
        gbs = byts / (ms / 1e3) / 1e9
        res[f"b{b}"] = {"us": round(ms * 1000, 2), "vectors_per_s": n / (ms / 1e3), "gbs": round(gbs, 1),
                        "frac_8tbs": round(gbs / HBM_NOMINAL_GBS, 4), "frac_measured": round(gbs / peak, 4)}
    del x
    torch.cuda.empty_cache()
    return res


def measure_config0(torch, tq, wl, reps=50):
    """Single head, d 128: 4096 fp32 keys (per-channel law, no per-token scale), 16 queries,
    b = 4 product code: absolute latency of tq_quantize and tq_logits (median of `reps`)."""
    d, n, nq = 128, 4096, 16
    x = torch.from_numpy(wl.head_vectors(n, d, seed=wl.SEED_KEYS, token_scale=False)).cuda()
    q = torch.from_numpy(wl.queries(nq, d)).cuda()
    p = tq.Params(d, 4, tq.TQ_MODE_PROD, 128, wl.SEED_PARAMS)
    c = torch.empty(p.code_bytes(n), dtype=torch.uint8, device="cuda")
    nn = torch.empty(n, dtype=torch.int16, device="cuda")
    rn = torch.empty(n, dtype=torch.int16, device="cuda")
    lg = torch.empty((nq, n), device="cuda")
    ws = torch.empty(tq.tq_logits_workspace(p, nq), dtype=torch.uint8, device="cuda")
    calls = {"tq_quantize": lambda: tq.tq_quantize(p, x, c, nn, rn),
             "tq_logits": lambda: tq.tq_logits(p, q, nq, c, nn, rn, n, 1, lg, ws)}
    res = {}
    for name, f in calls.items():
        for _ in range(5):
            f()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1000)
        res[name + "_us"] = round(statistics.median(ts), 2)
    res["workload"] = "single-head-4096x128-fp32-16q-b4"
    return res


def run_secondary(args, world, rank, local, torch, tq, wl):
    """Other workloads (their own JSON line): 'decode' = 64 sequences x 8 KV heads x 16384 tokens
    (K product b=3, V MSE b=3, 32 query heads); 'quantize' = 2^20 bf16 vectors at b=2,3,4;
    'search' = 10^4 queries over 10^6 vectors; 'polar' = the polar-coordinate code on the
    layer's keys (quantize + logits at w = 2, 3)."""
    peak, peak_kind = measured_peaks()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    if args.workload == "decode":
        r = measure_decode(torch, tq, wl, args.steps, args.warmup, peak, batch=args.decode_batch)
        n = args.decode_batch * 8 * 16384
        line = {"metric": "decode attention tokens/s", "value": r["tokens_per_s"], "unit": "tokens/s",
                "ms_per_step": r["us"] / 1000, "config": {"workload": r["workload"]}, "decode": r}
    elif args.workload == "quantize":
        res = measure_quantize(torch, tq, wl, args.steps, args.warmup, peak)
        line = {"metric": "quantize vectors/s", "value": res["b4"]["vectors_per_s"], "unit": "vectors/s",
                "config": {"workload": "quantize-2^20x128-bf16-prod-m128"}, "per_bits": res}
    elif args.workload == "polar":
        # polar-coordinate stage 1 on the layer's keys: 8 KV heads x 32768 tokens, d 128, bf16,
        # 32 query heads (GQA 4); quantize then logits, at w = 2 and 3 bits per coordinate
        H, T, d, G = 8, 32768, 128, 4
        n = H * T
        x = gpu_kv(torch, 1, H, T, d, wl.SEED_KEYS)
        q = torch.randn((H * G, d), device="cuda")
        calls, byts = [], {}
        for w in (2, 3):
            p = tq.PolarParams(d, w, seed=wl.SEED_PARAMS)
            c = torch.empty(p.code_bytes(n), dtype=torch.uint8, device="cuda")
            nn = torch.empty(n, dtype=torch.int16, device="cuda")
            lg = torch.empty((H * G, T), device="cuda")
            calls.append((f"polar_quantize_w{w}", lambda p=p, c=c, nn=nn: tq.tq_polar_quantize(p, x, c, nn)))
            calls.append((f"polar_logits_w{w}",
                          lambda p=p, c=c, nn=nn, lg=lg: tq.tq_polar_logits(p, q, G, c, nn, T, H, lg)))
            byts[f"polar_quantize_w{w}"] = n * d * 2 + c.numel() + 2 * n
            byts[f"polar_logits_w{w}"] = c.numel() + 2 * n + q.numel() * 4

        class _Calls:
            def calls(self):
                return calls
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
        step_ms, per_call = time_steps(torch, _Calls(), args.steps, args.warmup, world, flush)
        ms = statistics.median(step_ms)
        kern = {}
        for lab, ts in per_call.items():
            us = statistics.median(ts) * 1000
            gbs = byts[lab] / (us / 1e6) / 1e9
            kern[lab] = {"us": round(us, 2), "gbs": round(gbs, 1), "frac_measured": round(gbs / peak, 4)}
        line = {"metric": "polar-code keys/s (quantize + logits, w=2 and w=3)", "value": 2 * n / (ms / 1e3),
                "unit": "keys/s", "ms_per_step": ms,
                "config": {"workload": "polar-kv8x32768-gqa4-d128-bf16", "w": [2, 3],
                           "l2": "flushed between steps (256 MB write)"},
                "kernels": kern}
    elif args.workload == "project":
        # quantize-on-write: the K projection of one Llama-3.1-8B-shaped layer over a 32768-token
        # prefill (x [32768, 4096] bf16, W_k [8 * 128, 4096] bf16) coded in the same kernel, against
        # the unfused path (cuBLAS bf16 GEMM writing K, then tq_quantize per head)
        T, hid, H, d = 32768, 4096, 8, 128
        xnp, wnp = wl.projection_inputs(T, hid, H, wl.SEED_KEYS)
        x = torch.from_numpy(xnp).to(torch.bfloat16).cuda()
        w = torch.from_numpy(wnp).to(torch.bfloat16).cuda()
        del xnp, wnp
        n = H * T
        flops = 2.0 * T * hid * H * d
        bf16_peak = measured_bf16_peak()
        res = {}
        for b, mode in ((3, tq.TQ_MODE_PROD), (4, tq.TQ_MODE_PROD), (3, tq.TQ_MODE_MSE)):
            p = tq.Params(d, b, mode, 128 if mode == tq.TQ_MODE_PROD else 0, wl.SEED_PARAMS)
            c = torch.empty(p.code_bytes(n), dtype=torch.uint8, device="cuda")
            nn = torch.empty(n, dtype=torch.int16, device="cuda")
            rn = torch.empty(n, dtype=torch.int16, device="cuda") if mode == tq.TQ_MODE_PROD else None
            kbuf = torch.empty((T, H * d), dtype=torch.bfloat16, device="cuda")
            fused = lambda: tq.tq_project_quantize(p, x, w, H, c, nn, rn)

            def unfused():
                torch.matmul(x, w.T, out=kbuf)
                for h in range(H):
                    tq.tq_quantize(p, kbuf[:, h * d:(h + 1) * d], c[h * (p.code_bytes(T)):], nn[h * T:],
                                   rn[h * T:] if rn is not None else None, n_vec=T, ld=H * d)
            out = {}
            for lab, f in (("fused", fused), ("unfused", unfused)):
                for _ in range(max(3, args.warmup)):
                    f()
                torch.cuda.synchronize()
                e0, e1 = ev(), ev()
                e0.record()
                for _ in range(args.steps):
                    f()
                e1.record()
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1) / args.steps
                out[lab + "_us"] = round(ms * 1000, 1)
                out[lab + "_tflops"] = round(flops / (ms / 1e3) / 1e12, 1)
            out["frac_bf16_measured"] = round(out["fused_tflops"] * 1e12 / bf16_peak, 4)
            out["speedup_vs_unfused"] = round(out["unfused_us"] / out["fused_us"], 3)
            res[f"b{b}_{'prod' if mode == tq.TQ_MODE_PROD else 'mse'}"] = out
        line = {"metric": "quantize-on-write tokens/s (K projection + code, one layer)",
                "value": T / (res["b3_prod"]["fused_us"] / 1e6), "unit": "tokens/s",
                "config": {"workload": "llama3.1-8b-kproj-prefill-32768x4096-kv8", "bits": [3, 4],
                           "unfused": "torch.matmul (cuBLAS) writing K, then tq_quantize per head"},
                "per_bits": res}
    elif args.workload == "search":
        n_db, n_q, d, k = 1000000, 10000, 200, 10
        db = torch.from_numpy(wl.search_set(n_db, d, seed=wl.SEED_KEYS)).to(torch.bfloat16).cuda()
        qs = torch.from_numpy(wl.search_set(n_q, d, seed=wl.SEED_QUERIES)).cuda()
        # exact top-10 by fp32 inner product on the (bf16-rounded) database (torch.matmul, chunked)
        dbf = db.float()
        truth = []
        for s0 in range(0, n_q, 1000):
            sc = qs[s0:s0 + 1000] @ dbf.T
            truth.append(torch.topk(sc, k, dim=1).indices.cpu())
        truth = torch.cat(truth).numpy()
        del dbf
        res = {}
        for b in (2, 4):
            p = tq.Params(d, b, tq.TQ_MODE_PROD, 256, wl.SEED_PARAMS)
            c = torch.empty(p.code_bytes(n_db), dtype=torch.uint8, device="cuda")
            nn = torch.empty(n_db, dtype=torch.int16, device="cuda")
            rn = torch.empty(n_db, dtype=torch.int16, device="cuda")
            e0, e1 = ev(), ev()
            for _ in range(3):  # warm-up
                tq.tq_quantize(p, db, c, nn, rn)
            torch.cuda.synchronize()
            q_reps = 10
            e0.record()
            for _ in range(q_reps):
                tq.tq_quantize(p, db, c, nn, rn)
            e1.record()
            torch.cuda.synchronize()
            q_ms = e0.elapsed_time(e1) / q_reps
            ids = torch.empty((n_q, k), dtype=torch.int32, device="cuda")
            scs = torch.empty((n_q, k), dtype=torch.float32, device="cuda")
            ws = torch.empty(tq.tq_search_workspace(p, n_q, n_db, k), dtype=torch.uint8, device="cuda")
            run = lambda: tq.tq_search_topk(p, qs, c, nn, rn, n_db, k, ids, scs, ws)
            for _ in range(max(1, args.warmup)):
                run()
            torch.cuda.synchronize()
            e0.record()
            for _ in range(args.steps):
                run()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / args.steps
            got = ids.cpu().numpy()
            recall = float(np.mean([len(set(got[i]) & set(truth[i])) / k for i in range(n_q)]))
            q_bytes = n_db * d * 2 + c.numel() + 4 * n_db
            res[f"b{b}"] = {"search_ms": round(ms, 3), "estimates_per_s": n_q * n_db / (ms / 1e3),
                            "recall_at_10": round(recall, 4), "quantize_db_ms": round(q_ms, 3),
                            "quantize_db_gbs": round(q_bytes / (q_ms / 1e3) / 1e9, 1),
                            "quantize_db": "warm, mean of 10 calls after 3 warm-up calls"}
        line = {"metric": "search estimates/s", "value": res["b4"]["estimates_per_s"], "unit": "estimates/s",
                "config": {"workload": "search-1e6x200-1e4q-top10"}, "per_bits": res}
    else:
        raise SystemExit(f"workload {args.workload}: not available yet")
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- main
def layer_config(world):
    return {"workload": "llama3.1-8b-layer-kv8x32768-gqa4-d128", "kv_heads": 8, "tokens": 32768, "q_heads": 32,
            "d": 128, "bits": [3, 4], "kv_dtype": "bf16", "value": VALUE_DEF,
            "l2": "flushed between steps (256 MB write)", "parallelism": f"replicas x{world}"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    vals = []
    for _ in range(args.warmup):
        cpu_oracle_layer(sample_tokens=2048)
    for _ in range(max(1, args.steps)):
        v, cores, dt, sample = cpu_oracle_layer(sample_tokens=2048)
        vals.append(v)
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC,
            "value": v, "unit": "keys/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": layer_config(world),
            "cpu_baseline": {"value": v, "unit": "keys/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    world, rank, local = dist_setup(args)
    import vector_quantization_randomized_b200 as tq
    import workloads as wl
    if args.workload != "layer":
        return run_secondary(args, world, rank, local, torch, tq, wl)
    peak, peak_kind = measured_peaks()
    wk = Layer(tq, wl, torch)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    sampler = ClockSampler(local)
    sampler.start()
    step_ms, per_call = time_steps(torch, wk, args.steps, args.warmup, world, flush, sampler)
    clocks = sampler.stop()
    ms = statistics.mean(step_ms)
    ms_max = allmax(world, sum(step_ms)) / args.steps
    value = weak_scaling_value(world, wk.keys_per_step(), ms_max)

    # dominant API call in the step and its roofline
    kinds = {}
    for label, times in per_call.items():
        kind = label.rsplit("_b", 1)[0]
        k = kinds.setdefault(kind, [0.0, 0.0, 0])
        k[0] += sum(times)
        k[1] += wk.bytes_of(label) * len(times)
        k[2] += len(times)
    dom = max(kinds, key=lambda k: kinds[k][0])
    t_ms, byts, nl = kinds[dom]
    achieved = byts / (t_ms / 1e3) / 1e9
    traffic = traffic_record(dom)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": dom,
                "peak_kind": f"{peak_kind} (copy bandwidth)", "algorithmic_bytes_per_launch": int(byts / nl)}

    kernels = {}
    for label, times in per_call.items():
        avg = statistics.mean(times)
        gbs = wk.bytes_of(label) / (avg / 1e3) / 1e9
        kernels[label] = {"us": round(avg * 1000, 2), "gbs": round(gbs, 1), "frac_measured": round(gbs / peak, 4)}
    logits = None
    if not args.no_kernels:
        iso = logits_isolated(torch, tq, wk)
        logits = {}
        for b, (us, mb, lat) in iso.items():
            gbs = mb / (us / 1e6) / 1e9
            kernels[f"tq_logits_b{b}_l2cold"] = {
                "us": round(us, 2), "keys_per_s": round(wk.n / (us / 1e6)), "gbs": round(gbs, 1),
                "frac_8tbs": round(gbs / HBM_NOMINAL_GBS, 4), "frac_measured": round(gbs / peak, 4),
                "single_launch_us": round(lat, 2)}
            logits[f"b{b}"] = {"keys_per_s": round(wk.n / (us / 1e6)), "gbs": round(gbs, 1),
                               "frac_8tbs": round(gbs / HBM_NOMINAL_GBS, 4), "frac_measured": round(gbs / peak, 4),
                               "us_per_call": round(us, 2), "metric_bytes": int(mb)}
        logits["how"] = ("tq_logits alone (query preparation included), one call per distinct copy of the codes; "
                         f"copies total > 4x L2, launches captured in a CUDA graph")

    configs = None
    if not args.no_configs:
        configs = {"config0_latency": measure_config0(torch, tq, wl),
                   "quantize_2^20": measure_quantize(torch, tq, wl, max(5, args.steps // 2), 3, peak),
                   "decode": measure_decode(torch, tq, wl, max(5, args.steps // 2), 3, peak, sparse=False)}

    e2e = None
    if not args.no_e2e:
        e_ms, h2d, d2h = time_e2e(torch, wk, max(3, args.steps // 2), 2)
        e_ms = allmax(world, e_ms)
        e2e = {"value": weak_scaling_value(world, wk.keys_per_step(), e_ms), "unit": "keys/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        v, cores, dt, sample = cpu_oracle_layer()
        cpu = {"value": v, "unit": "keys/s", "cores": cores, "kind": "oracle", "sample": sample,
               "seconds": round(dt, 2), "one_core": cpu_oracle_one_core()}
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "keys/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32+s8",
                "data": "synthetic",
                "config": layer_config(world),
                "roofline": roofline, "logits": logits, "kernels": kernels, "configs": configs,
                "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": wk.launches_per_step * args.steps, "clocks": clocks}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
