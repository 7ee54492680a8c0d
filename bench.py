"""Benchmark of the sigmoid-routed MoE block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = route + permute + expert up-projection + down-projection + combine
over one batch of synthetic tokens (the whole hot path), inputs resident in HBM.
Default workload: the GLM-5-shaped prefill block (16384 tokens, H 6144, 256
experts top-8 + 1 shared, I 2048).  Prints ONE JSON line on rank 0.

N > 1 runs independent replicas, one per GPU (the layer has no cross-token
term, so each rank processes its own batch; no data-path collective): weak
scaling, value = tokens of all ranks / max over ranks of the device time.

--impl reference times the CPU oracle (the slow, plain statement of the
method, double precision, OpenMP) on the host cores, each step a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
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

from sigmoid_routed_mixture_b200 import workloads as W  # noqa: E402

METRIC = "MoE-block tokens/s (GLM-5 shape, bf16, 1 B200)"
UNIT = "tokens/s"
KERNELS_PER_DENSE_STEP = 4  # identity rows 1 + up 1 + down 1 + combine 1


def kernels_per_step(w, num_sms=148):
    """Kernel launches of one routed step: the router (one kernel: logits,
    selection and gates, with the router weights split once at pack time);
    permutation (one CTA for small batches, one launch over at most one
    1024-assignment chunk per SM, else histogram + scan + scatter); token gather
    (invert + scatter); up GEMM; down GEMM; combine."""
    route = 1
    n = w.T * w.K
    permute = 1 if n <= 4096 or -(-n // 1024) <= num_sms else 3
    return route + permute + 2 + 1 + 1 + 1


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return dict(hbm=float(p["hbm_gbs"]), tflops=float(p["bf16_tflops"]),
                    tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, tflops=1590.0, tflops_sustained=1400.0, source="fallback")


def tensor_peak(pk, timed_loop_ms):
    """The bf16 peak a tensor-bound kernel is judged against: the sustained
    figure (cuBLAS back to back for seconds, under the board power cap) when the
    kernel was timed inside a timed loop of at least half a second, else the
    burst figure (a kernel timed alone).  Returns (TFLOP/s, description)."""
    if timed_loop_ms >= 500.0:
        return pk["tflops_sustained"], "sustained bf16 (cuBLAS back to back), %s; timed loop %.2f s" % (
            pk["source"], timed_loop_ms / 1e3)
    return pk["tflops"], "burst bf16 (cuBLAS), %s; timed loop %.2f s" % (pk["source"], timed_loop_ms / 1e3)


# ------------------------------------------------------------------ clocks

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, device_index: int):
        self.tmp = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        self.proc = None
        self.dev = device_index

    def start(self):
        try:
            ids = os.environ.get("CUDA_VISIBLE_DEVICES")
            gpu = ids.split(",")[self.dev] if ids else str(self.dev)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + CLOCK_FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", gpu], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        rows = [r.split(",") for r in open(self.tmp.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.tmp.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ oracle sample

def oracle_sample_tokens(w, counts_of_token_experts, n_tokens, max_experts=48):
    """Token sample for the CPU oracle: tokens whose K experts all lie among the
    `max_experts` most loaded ones (bounds the weights the host must hold; the
    oracle's cost per token does not depend on which experts it uses)."""
    idx = counts_of_token_experts
    load = np.bincount(idx.reshape(-1), minlength=w.E)
    top = set(np.argsort(-load)[:max_experts].tolist())
    cand = [t for t in range(idx.shape[0]) if set(idx[t].tolist()) <= top]
    if len(cand) < n_tokens:
        cand = list(range(min(n_tokens, idx.shape[0])))
    return np.array(cand[:n_tokens], dtype=np.int64)


def run_oracle_steps(w, x, w_r, b, tokens, expert_tables, shared, steps):
    """Time route + permute + forward of the oracle on `tokens`, `steps` times."""
    from oracle import oracle as O

    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        idx, gate, margin, z = O.route(x[tokens], w_r, b, w.K, w.scale)
        O.permute(idx, w.E, w.has_shared)
        O.forward(x[tokens], expert_tables[0], expert_tables[1], expert_tables[2], shared[0], shared[1],
                  shared[2], idx, gate, has_shared=w.has_shared)
        times.append(time.perf_counter() - t0)
    return times


def host_expert_tables(w, experts, getter):
    t1 = [getter("w1", e) if e in experts else None for e in range(w.E)]
    t3 = [getter("w3", e) if e in experts else None for e in range(w.E)]
    t2 = [getter("w2", e) if e in experts else None for e in range(w.E)]
    return t1, t3, t2


def cores():
    return len(os.sched_getaffinity(0))


def kernel_source_hash(kernel):
    """md5 of the sources a kernel's DRAM traffic depends on: the grouped GEMM
    (grouped_gemm.cu, common.cuh, the GemmArgs block of kernels.h) or the key
    selection's score kernel (its section of dsa.cu, common.cuh)."""
    import hashlib

    h = hashlib.md5()
    csrc = os.path.join(ROOT, "sigmoid_routed_mixture_b200", "csrc")
    if kernel.startswith("dsa_score"):
        h.update(open(os.path.join(csrc, "common.cuh"), "rb").read())
        src = open(os.path.join(csrc, "dsa.cu"), "rb").read()
        a = src.index(b"// ---------------------------------------------------------------- 2) scores")
        b = src.index(b"// ---------------------------------------------------------------- 3) top-k")
        h.update(src[a:b])
        return h.hexdigest()
    h.update(open(os.path.join(csrc, "grouped_gemm.cu"), "rb").read())
    h.update(open(os.path.join(csrc, "common.cuh"), "rb").read())
    hdr = open(os.path.join(csrc, "kernels.h"), "rb").read()
    a = hdr.index(b"struct GemmArgs {")
    h.update(hdr[a:hdr.index(b"};", a) + 2])  # the GEMM's argument block, not the other declarations
    return h.hexdigest()


def measured_traffic(workload, kernel):
    """DRAM bytes per launch from a committed ncu capture (the `traffic` lines of
    the profile summaries), or None when the kernel's sources changed since it
    was taken."""
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    want = "src=" + kernel_source_hash(kernel)
    for fn in sorted(os.listdir(pdir)):
        if not fn.endswith(".md"):
            continue
        for line in open(os.path.join(pdir, fn)):
            parts = line.split()
            if len(parts) == 5 and parts[0] == "traffic" and parts[1] == workload and parts[2] == kernel:
                if parts[4] == want:
                    return float(parts[3])
    return None


# ------------------------------------------------------------------ reference arm

def run_reference(args, rank):
    if rank != 0:
        return
    os.environ.setdefault("OMP_NUM_THREADS", str(cores()))
    from oracle import oracle as O

    O.build()
    w = W.WORKLOADS[args.workload]
    x, w_r, b = W.router_inputs(w)
    idx, _, _, _ = O.route(x[: min(w.T, 4096)], w_r, b, w.K, w.scale)
    n = max(1, min(args.ref_tokens or 2 * cores(), w.T))
    tokens = oracle_sample_tokens(w, idx, n)
    sel, _, _, _ = O.route(x[tokens], w_r, b, w.K, w.scale)
    experts = set(np.unique(sel).tolist())
    rng_cache = {}

    def getter(name, e):  # host-generated bf16 weights of the sampled experts (N(0, 0.02))
        key = (name, e)
        if key not in rng_cache:
            rng = np.random.default_rng([w.seed, ("w1", "w3", "w2").index(name), e])
            shape = (w.I, w.H) if name != "w2" else (w.H, w.I)
            rng_cache[key] = W.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(0.02))
        return rng_cache[key]

    tables = host_expert_tables(w, experts, getter)
    rng = np.random.default_rng([w.seed, 9])
    shared = [W.f32_to_bf16_bits(rng.standard_normal(s, dtype=np.float32) * np.float32(0.02))
              for s in ((w.I, w.H), (w.I, w.H), (w.H, w.I))]
    run_oracle_steps(w, x, w_r, b, tokens, tables, shared, args.warmup)
    times = run_oracle_steps(w, x, w_r, b, tokens, tables, shared, args.steps)
    total = sum(times)
    value = len(tokens) * args.steps / total
    sample = ("route+permute+forward of %d of the %d tokens per step (double-precision C oracle, "
              "OpenMP), %d distinct experts" % (len(tokens), w.T, len(experts)))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": workload_config(w, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(os.environ["OMP_NUM_THREADS"]),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ replicas (N > 1)

def replica_tokens(w, rank):
    """Token batch of replica `rank`: the workload's own x on rank 0, an
    independently seeded batch of the same shape on the others."""
    x, w_r, b = W.router_inputs(w)
    if rank > 0:
        rng = np.random.default_rng([w.seed, rank])
        x = W.f32_to_bf16_bits(rng.standard_normal(x.shape, dtype=np.float32))
        if w.skew:
            x[:, 0] = W.f32_to_bf16_bits(np.ones((w.T,), dtype=np.float32))
    return x, w_r, b


def pipelined_e2e(torch, stream, dev, n_steps, dist, copy_in, replays, copy_out):
    """Device time (max over ranks) of n_steps end-to-end steps, each made of its
    input copy (host -> device, copy_in(j)), its compute (replays[j]() on `stream`)
    and its output copy (device -> host, copy_out(j)), for the buffer set
    j = step % 2.  The copies run on their own streams, so step i + 1's input
    and step i - 1's output move while step i computes; the events keep a
    buffer set from being refilled before its compute and output copy are done."""
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            j = i % 2
            if i >= 2:
                h2d.wait_event(ev_comp[j])
            with torch.cuda.stream(h2d):
                copy_in(j)
                ev_in[j].record(h2d)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])
            replays[j]()
            ev_comp[j].record(stream)
            d2h.wait_event(ev_comp[j])
            with torch.cuda.stream(d2h):
                copy_out(j)
                ev_out[j].record(d2h)

    run(2)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    z = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    a.record(h2d)
    run(n_steps)
    z.record(d2h)
    torch.cuda.synchronize()
    return max_over_ranks(a.elapsed_time(z), dist, dev)


def max_over_ranks(ms, dist, device):
    """The slowest replica's device time (every rank takes the same collective)."""
    if dist is None:
        return ms
    import torch

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(tokens_per_rank, world, steps, t_max_ms):
    """Whole-job throughput: tokens of all replicas over the slowest replica's time."""
    return tokens_per_rank * world * steps / (t_max_ms / 1e3)


class DenseBlock:
    """The dense SwiGLU MLP of the first blocks with its buffers (bench only)."""

    def __init__(self, cfg, weights, dev):
        import torch
        from sigmoid_routed_mixture_b200 import moe

        self.cfg = cfg
        self.weights = weights
        self.ws = moe.workspace(cfg, device=dev)
        self.y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
        self.counts = torch.zeros((1,), dtype=torch.int32, device=dev)
        self.margin = torch.ones((cfg.T,), dtype=torch.float32, device=dev)

    def __call__(self, x):
        from sigmoid_routed_mixture_b200 import moe

        return moe.dense_mlp(self.cfg, self.weights, x, self.ws, y=self.y)


def workload_config(w, args):
    return {"workload": w.name, "tokens": w.T, "hidden": w.H, "expert_intermediate": w.I,
            "routed_experts": w.E, "top_k": w.K, "shared_experts": int(w.has_shared),
            "routed_scale": w.scale, "skewed_routing": w.skew, "global_batch": w.T * args.gpus,
            "parallelism": "replicas x%d" % args.gpus,
            "l2": "inputs larger than L2 (packed expert weights %.1f GB)" % (
                (w.E + 1) * 3 * w.H * w.I * 2 / 1e9)}


# ------------------------------------------------------------------ key selection workloads

DSA_METRIC = "DSA key selections/s (GLM-5 indexer, 32 heads x 128, top-2048, 1 B200)"
DSA_UNIT = "queries/s"
DSA_KERNELS_PER_STEP = 3  # plan, scores, top-k


def dsa_visible_pairs(w):
    """(query, key) pairs the causal mask leaves: sum over queries of S - T + t + 1."""
    return w.B * (w.T * (w.S - w.T) + w.T * (w.T + 1) // 2)


def dsa_replica_inputs(w, rank):
    """(q, k, w) of replica `rank`: the workload's own inputs on rank 0, an
    independently seeded draw of the same shapes on the others."""
    return W.dsa_inputs(w if rank == 0 else w.replace(seed=w.seed + 7919 * rank))


def dsa_oracle_sample(w, n, inputs):
    """A bounded oracle sample: n consecutive queries of sequence 0 around the
    middle of the prompt (prefill), or the single query of n sequences (decode).
    Returns (seconds, queries)."""
    from oracle import oracle as O

    q, k, wt = inputs
    if w.T == 1:
        n = min(n, w.B)
        t0 = time.time()
        O.dsa_select(O.dsa_scores(q[:n], k[:n], wt[:n]), w.topk)
        return time.time() - t0, n
    n = min(n, w.T)
    p = min(w.T - 1, (w.S - w.T) + w.T // 2 + n // 2)  # position of the last sampled query
    t_hi = p - (w.S - w.T)
    qs, ws_ = q[:1, t_hi - n + 1:t_hi + 1], wt[:1, t_hi - n + 1:t_hi + 1]
    t0 = time.time()
    O.dsa_select(O.dsa_scores(qs, k[:1, :p + 1], ws_), w.topk)
    return time.time() - t0, n


def dsa_line_config(w, world):
    return {"workload": w.name, "sequences": w.B, "queries_per_sequence": w.T, "keys_per_sequence": w.S,
            "index_heads": w.n_heads, "index_head_dim": w.head_dim, "topk": w.topk,
            "global_batch": w.B * w.T * world, "parallelism": "replicas x%d" % world,
            "l2": "inputs larger than L2: q %.0f MB, keys %.0f MB and scores %.0f MB per step against 126 MB" % (
                w.B * w.T * w.n_heads * w.head_dim * 2 / 1e6, w.B * w.S * w.head_dim * 2 / 1e6,
                dsa_visible_pairs(w) * 4 / 1e6)}


def run_dsa_reference(args, rank):
    if rank != 0:
        return
    os.environ.setdefault("OMP_NUM_THREADS", str(cores()))
    from oracle import oracle as O

    O.build()
    w = W.DSA_WORKLOADS[args.workload]
    n = args.ref_tokens or 2 * cores()
    inputs = W.dsa_inputs(w)
    for _ in range(args.warmup):
        dsa_oracle_sample(w, n, inputs)
    secs, nq = 0.0, 0
    for _ in range(args.steps):
        s_, q_ = dsa_oracle_sample(w, n, inputs)
        secs += s_
        nq += q_
    value = nq / secs
    sample = "scores + top-%d of %d queries per step (double-precision C oracle, OpenMP)" % (w.topk, nq // args.steps)
    line = {"impl": "reference", "metric": DSA_METRIC, "value": value, "unit": DSA_UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": dsa_line_config(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": DSA_UNIT, "cores": int(os.environ["OMP_NUM_THREADS"]),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": DSA_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_dsa(args, world, rank, dist, dev):
    import torch

    from sigmoid_routed_mixture_b200 import dsa, moe

    w = W.DSA_WORKLOADS[args.workload]
    q, k, wt = dsa_replica_inputs(w, rank)
    cfg = dsa.Config(w.B, w.T, w.S, w.n_heads, w.head_dim, w.topk)
    ws = dsa.workspace(cfg, device=dev)
    q_dev = torch.from_numpy(q.view(np.int16)).to(dev).view(torch.bfloat16)
    k_dev = torch.from_numpy(k.view(np.int16)).to(dev).view(torch.bfloat16)
    w_dev = torch.from_numpy(wt).to(dev)
    scores = torch.empty((w.B, w.T, w.S), dtype=torch.float32, device=dev)
    sel = torch.empty((w.B, w.T, cfg.n_sel), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None, bufs=None):
        qd, kd, wd, sd = bufs if bufs is not None else (q_dev, k_dev, w_dev, sel)
        if ev is not None:
            ev[0].record(stream)
        dsa.scores(cfg, qd, kd, wd, ws, out=scores)
        if ev is not None:
            ev[1].record(stream)
        dsa.topk(cfg, scores, ws, out=sd)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if moe.device_error(ws) != 0:
        raise RuntimeError("device error during warm-up")
    graph = None
    if not args.eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(args.warmup):
            graph.replay()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch.cuda.current_device())
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    e0.record(stream)
    for i in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step(evs[i])
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    total_ms = e0.elapsed_time(e1)
    if graph is not None:  # stage breakdown from host-launched steps after the timed ones
        for i in range(args.steps):
            step(evs[i])
        torch.cuda.synchronize()
    stage = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(2)] for i in range(args.steps)])
    t_max = max_over_ranks(total_ms, dist, dev)
    value = w.B * w.T * world * args.steps / (t_max / 1e3)

    # end to end: q, k, w from pinned host memory in, the selection out, every
    # step; two buffer sets and copy streams overlap the copies with the compute
    hq = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).pin_memory()
    hk = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16).pin_memory()
    hw = torch.from_numpy(wt).pin_memory()
    hsel = [torch.empty(tuple(sel.shape), dtype=torch.int32).pin_memory() for _ in range(2)]
    bufs = [(q_dev, k_dev, w_dev, sel),
            (torch.empty_like(q_dev), torch.empty_like(k_dev), torch.empty_like(w_dev), torch.empty_like(sel))]
    replays = []
    for j in range(2):
        if graph is not None and j == 0:
            replays.append(graph.replay)
        elif graph is not None:
            step(bufs=bufs[1])
            torch.cuda.synchronize()
            g1 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g1):
                step(bufs=bufs[1])
            replays.append(g1.replay)
        else:
            replays.append(lambda j=j: step(bufs=bufs[j]))

    def copy_in(j):
        bufs[j][0].copy_(hq, non_blocking=True)
        bufs[j][1].copy_(hk, non_blocking=True)
        bufs[j][2].copy_(hw, non_blocking=True)

    e2e_ms = pipelined_e2e(torch, stream, dev, args.e2e_steps, dist, copy_in, replays,
                           lambda j: hsel[j].copy_(bufs[j][3], non_blocking=True))
    if moe.device_error(ws) != 0:
        raise RuntimeError("device error during the timed steps")

    pk = peaks()
    pairs = dsa_visible_pairs(w)
    f_score = 2.0 * pairs * w.n_heads * w.head_dim
    b_in = w.B * w.T * w.n_heads * w.head_dim * 2 + w.B * w.S * w.head_dim * 2 + w.B * w.T * w.n_heads * 4
    b_sel = w.B * w.T * cfg.n_sel * 4
    b_score = b_in + pairs * 4       # inputs + the scores it writes
    b_topk = pairs * 4 + b_sel       # the visible scores read + the selection written
    mean = stage.mean(axis=0)
    tpk, tpk_kind = tensor_peak(pk, total_ms)
    ridge = tpk * 1e12 / (pk["hbm"] * 1e9)
    kernels = [("dsa_score_kernel", f_score, b_score, mean[0]), ("dsa_topk_kernel", 0.0, b_topk, mean[1])]
    name, f, by, ms = max(kernels, key=lambda x: x[3])
    if f > 0 and f / by > ridge:
        roof = {"kernel": name, "bound": "tensor", "achieved": f / (ms / 1e3) / 1e12, "peak": tpk,
                "unit": "TFLOP/s", "peak_kind": tpk_kind, "algorithmic_per_launch": f}
    else:
        roof = {"kernel": name, "bound": "hbm", "achieved": by / (ms / 1e3) / 1e9, "peak": pk["hbm"],
                "unit": "GB/s", "peak_kind": "copy bandwidth, " + pk["source"], "algorithmic_per_launch": by}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = measured_traffic(w.name, name)
    step_s = t_max / 1e3 / args.steps
    t_roof = max(f_score / (tpk * 1e12), (b_in + b_sel) / (pk["hbm"] * 1e9))
    line = {
        "metric": DSA_METRIC, "value": value, "unit": DSA_UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded q, k, w of the GLM-5 indexer shapes)",
        "config": dsa_line_config(w, world), "roofline": roof,
        "block_roofline": {"t_roof_ms": t_roof * 1e3, "frac": t_roof / step_s, "f_alg_tflop": f_score / 1e12,
                           "b_alg_gb": (b_in + b_sel) / 1e9},
        "stage_ms": {"scores": float(mean[0]), "topk": float(mean[1])},
        "stage_roofline": {
            "scores": {"bound": "tensor" if f_score / b_score > ridge else "hbm",
                       "frac": (f_score / (mean[0] / 1e3) / 1e12 / tpk) if f_score / b_score > ridge
                       else (b_score / (mean[0] / 1e3) / 1e9 / pk["hbm"])},
            "topk": {"bound": "hbm", "frac": b_topk / (mean[1] / 1e3) / 1e9 / pk["hbm"]}},
        "launch": "cuda graph replay" if graph is not None else "eager",
        "e2e": {"value": w.B * w.T * world * args.e2e_steps / (e2e_ms / 1e3), "unit": DSA_UNIT,
                "h2d_bytes_per_step": int(b_in), "d2h_bytes_per_step": int(b_sel), "steps": args.e2e_steps,
                "copies": "pinned host buffers, H2D and D2H on their own streams overlapping the compute of the "
                          "neighbouring steps (two device buffer sets)"},
        "gpu_launches": DSA_KERNELS_PER_STEP * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        os.environ.setdefault("OMP_NUM_THREADS", str(cores()))
        from oracle import oracle as O

        O.build()
        secs, nq = dsa_oracle_sample(w, args.cpu_tokens or 2 * cores(), (q, k, wt))
        reps = 1
        while secs < 10.0 and secs * (reps + 1) / reps < 30.0:  # about 10 s of oracle work
            s_, q_ = dsa_oracle_sample(w, args.cpu_tokens or 2 * cores(), (q, k, wt))
            secs += s_
            nq += q_
            reps += 1
        line["cpu_baseline"] = {"value": nq / secs, "unit": DSA_UNIT, "cores": int(os.environ["OMP_NUM_THREADS"]),
                                "kind": "oracle",
                                "sample": "scores + top-%d of %d queries, %d times (double-precision C oracle, "
                                          "OpenMP), %.1f s" % (w.topk, nq // reps, reps, secs)}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ router stage

ROUTER_WORKLOADS = {"router_glm5_prefill": "glm5_prefill", "router_glm5_decode": "glm5_decode",
                    "router_glm47flash": "glm47flash"}


def router_metric(w):
    shape = "GLM-5 shape" if w.name.startswith("glm5") else "GLM-4.7-Flash shape"
    return "router tokens/s (%s: %d experts top-%d, H %d, 1 B200)" % (shape, w.E, w.K, w.H)


def run_router(args, world, rank, dist, dev):
    """The router alone (moe_route_packed: logits, scores, biased top-K, margin,
    gates in one kernel) on the block's tokens, timed like the block: CUDA-graph
    replays between device synchronisations, CUDA events.  Roofline: the split
    logits' tensor-core work (3 x 2 T H E_pad FLOP; the algorithmic 2 T H E is
    given too) against the bf16 peak, the bytes (x, W_r split, outputs) against
    HBM."""
    import torch

    from sigmoid_routed_mixture_b200 import moe

    w = W.WORKLOADS[ROUTER_WORKLOADS[args.workload]]
    x, w_r, b = replica_tokens(w, rank)
    cfg = moe.Config.of(w)
    x_dev = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    w_r_dev, b_dev = torch.from_numpy(w_r).to(dev), torch.from_numpy(b).to(dev)
    packed = moe.pack_router(cfg, w_r_dev)
    ws = moe.workspace(cfg, device=dev)
    out = moe.route_packed(cfg, x_dev, packed, b_dev, ws)
    stream = torch.cuda.current_stream()

    def step():
        moe.route_packed(cfg, x_dev, packed, b_dev, ws, out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(args.warmup):
        graph.replay()
    sampler = ClockSampler(torch.cuda.current_device())
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    a.record(stream)
    for _ in range(args.steps):
        graph.replay()
    z.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if moe.device_error(ws) != 0:
        raise RuntimeError("device error during the timed steps")
    t_max = max_over_ranks(a.elapsed_time(z), dist, dev)
    ms = t_max / args.steps
    pk = peaks()
    e_pad = -(-w.E // 64) * 64
    f_split = 3 * 2.0 * w.T * w.H * e_pad
    f_alg = 2.0 * w.T * w.H * w.E
    bytes_ = w.T * w.H * 2 + 3 * e_pad * w.H * 2 + w.E * 4 + w.T * w.K * 8 + w.T * 4
    tpk, tpk_kind = tensor_peak(pk, t_max)
    t_roof = max(f_split / (tpk * 1e12), bytes_ / (pk["hbm"] * 1e9))
    if f_split / (tpk * 1e12) >= bytes_ / (pk["hbm"] * 1e9):
        roof = {"kernel": "router_kernel", "bound": "tensor", "achieved": f_split / (ms / 1e3) / 1e12, "peak": tpk,
                "unit": "TFLOP/s", "peak_kind": tpk_kind, "algorithmic_per_launch": f_split}
    else:
        roof = {"kernel": "router_kernel", "bound": "hbm", "achieved": bytes_ / (ms / 1e3) / 1e9, "peak": pk["hbm"],
                "unit": "GB/s", "peak_kind": "copy bandwidth, " + pk["source"], "algorithmic_per_launch": bytes_}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = None
    line = {"metric": router_metric(w), "value": w.T * world * args.steps / (t_max / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 x, fp32 W_r (3-part split)",
            "data": "synthetic (seeded)", "config": dict(workload_config(w, argparse.Namespace(gpus=world)),
                                                         workload=args.workload),
            "roofline": roof, "router_roofline": {"t_roof_ms": t_roof * 1e3, "frac": t_roof / (ms / 1e3),
                                                  "f_split_tflop": f_split / 1e12, "f_alg_tflop": f_alg / 1e12,
                                                  "bytes_gb": bytes_ / 1e9},
            "launch": "cuda graph replay", "gpu_launches": args.steps, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

STAGES = ["route", "permute", "gather_tokens", "expert_up", "expert_down", "combine"]


def build_step(cfg, blk, x_dev, dense, stream):
    """One pass of the hot path on `stream`; with `ev` (7 events) it records the
    stage boundaries.  xin / yout replace the block's input and output buffers."""
    from sigmoid_routed_mixture_b200 import moe

    def step(ev=None, xin=None, yout=None):
        xin = x_dev if xin is None else xin
        yout = blk.y if yout is None else yout
        if dense:
            # one stage: the dense MLP (identity rows, up, down, combine)
            if ev is not None:
                for j in range(4):
                    ev[j].record(stream)
            moe.dense_mlp(cfg, blk.weights, xin, blk.ws, y=yout)
            if ev is not None:
                for j in range(4, 7):
                    ev[j].record(stream)
            return
        if ev is not None:
            ev[0].record(stream)
        moe.route_packed(cfg, xin, blk.router_packed, blk.bias, blk.ws, out=(blk.idx, blk.gate, blk.margin))
        if ev is not None:
            ev[1].record(stream)
        moe.permute(cfg, blk.idx, blk.ws, out=(blk.counts, blk.offsets, blk.sorted))
        if ev is not None:
            ev[2].record(stream)
        moe.gather_tokens(cfg, xin, blk.sorted, blk.ws)
        if ev is not None:
            ev[3].record(stream)
        moe.expert_up(cfg, blk.weights, blk.offsets, blk.sorted, blk.ws)
        if ev is not None:
            ev[4].record(stream)
        moe.expert_down(cfg, blk.weights, blk.gate, blk.offsets, blk.sorted, blk.ws)
        if ev is not None:
            ev[5].record(stream)
        moe.combine(cfg, blk.ws, yout)
        if ev is not None:
            ev[6].record(stream)

    return step


def measure_block(step, ws, steps, warmup, eager, dist, stream):
    """Warm-up, then EXACTLY `steps` timed steps (CUDA-graph replays, or host
    launches with `eager`) between a barrier and device synchronisations, with
    the SM clocks sampled meanwhile; then the same number of host-launched
    steps with events at the stage boundaries (they only feed the stage shares
    and the kernel roofline).  Returns a dict of the timings and the graph."""
    import torch

    from sigmoid_routed_mixture_b200 import moe

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if moe.device_error(ws) != 0:
        raise RuntimeError("device error during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(steps)]
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch.cuda.current_device())
    graph = None
    if not eager:
        # the step captured once as a CUDA graph and replayed: every kernel of
        # every step still runs; only the host launch gaps go away
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(warmup):
            graph.replay()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    e_start.record(stream)
    for i in range(steps):
        if graph is not None:
            graph.replay()
        else:
            step(evs[i])
    e_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if dist is not None:
        dist.barrier()
    total_ms = e_start.elapsed_time(e_end)
    eager_ms = total_ms
    if graph is not None:
        e_start.record(stream)
        for i in range(steps):
            step(evs[i])
        e_end.record(stream)
        torch.cuda.synchronize()
        eager_ms = e_start.elapsed_time(e_end)
    stage_ms = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(6)] for i in range(steps)])
    if moe.device_error(ws) != 0:
        raise RuntimeError("device error during the timed steps")
    return dict(graph=graph, total_ms=total_ms, eager_ms=eager_ms, stage_ms=stage_ms, clocks=clocks)


def block_record(w, cfg, blk, meas, t_max, steps, pk, dense):
    """Roofline of the dominant kernel, the block roofline and the routing
    statistics of one measured block (the algorithmic work of the method, from
    this run's own expert counts)."""
    counts = blk.counts.cpu().numpy()
    touched = (int((counts[: w.E] > 0).sum()) if not dense else 0) + int(w.has_shared)
    rows = cfg.rows
    H, I = w.H, w.I
    f_router = 2.0 * w.T * H * w.E
    f_up = 2.0 * rows * H * 2 * I
    f_down = 2.0 * rows * I * H
    # algorithmic bytes: weights of the touched groups plus the block's own
    # input (x) or output (y); intermediates (gathered rows, h, slot outputs)
    # are implementation choices and are not counted
    b_up = touched * 2 * I * H * 2 + w.T * H * 2
    b_down = touched * H * I * 2 + w.T * H * 2
    mean_stage = meas["stage_ms"].mean(axis=0)
    names = list(STAGES)
    if dense:
        names[3] = "dense_mlp"
    dom = int(np.argmax(mean_stage))
    tpk, tpk_kind = tensor_peak(pk, meas["total_ms"])
    ridge = tpk * 1e12 / (pk["hbm"] * 1e9)
    work = {"expert_up": (f_up, b_up), "expert_down": (f_down, b_down),
            "route": (f_router, w.T * H * 2 + w.E * H * 4 + w.T * w.K * 8),
            "permute": (0.0, w.T * w.K * 4 * 3 + rows * 4),
            "gather_tokens": (0.0, w.T * H * 2 + rows * H * 2),
            "combine": (0.0, rows * H * 2 + w.T * H * 2),
            "dense_mlp": (f_up + f_down, 3 * H * I * 2 + 2 * w.T * H * 2)}
    f, by = work[names[dom]]
    dur_s = mean_stage[dom] / 1e3
    if f > 0 and f / by > ridge:
        roof = {"kernel": names[dom], "bound": "tensor", "achieved": f / dur_s / 1e12,
                "peak": tpk, "unit": "TFLOP/s", "peak_kind": tpk_kind,
                "frac_of_burst": f / dur_s / 1e12 / pk["tflops"]}
    else:
        roof = {"kernel": names[dom], "bound": "hbm", "achieved": by / dur_s / 1e9, "peak": pk["hbm"],
                "unit": "GB/s", "peak_kind": "copy bandwidth, " + pk["source"]}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = measured_traffic(w.name, names[dom])
    roof["algorithmic_per_launch"] = f if roof["bound"] == "tensor" else by
    f_alg = f_router + f_up + f_down
    b_alg = touched * 3 * H * I * 2 + w.E * H * 4 + w.E * 4 + 2 * w.T * H * 2
    step_s = t_max / 1e3 / steps
    t_roof = max(f_alg / (tpk * 1e12), b_alg / (pk["hbm"] * 1e9))
    return {
        "roofline": roof,
        "block_roofline": {"t_roof_ms": t_roof * 1e3, "frac": t_roof / step_s,
                           "bound": "tensor" if f_alg / (tpk * 1e12) >= b_alg / (pk["hbm"] * 1e9) else "hbm",
                           "f_alg_tflop": f_alg / 1e12, "b_alg_gb": b_alg / 1e9},
        "stage_ms": {n: float(v) for n, v in zip(names, mean_stage)},
        "routing": None if dense else {
            "touched_groups": touched, "zero_count_experts": int((counts[: w.E] == 0).sum()),
            "max_count": int(counts[: w.E].max()), "min_count": int(counts[: w.E].min()),
            "near_ties": int((blk.margin <= 1e-4).sum().item())},
    }


def steps_for(step, stream, target_ms=250.0, lo=20, hi=4000):
    """Steps whose timed loop lasts about target_ms (estimated from 5 host-launched steps)."""
    import torch

    a = torch.cuda.Event(enable_timing=True)
    z = torch.cuda.Event(enable_timing=True)
    step()
    a.record(stream)
    for _ in range(5):
        step()
    z.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(z) / 5
    return int(min(hi, max(lo, -(-target_ms // max(ms, 1e-3)))))


def also_records(args, dev, stream, pk, packed):
    """The other block configurations, each timed like the headline (CUDA-graph
    replays, >= 0.25 s of timed loop, clocks sampled): the 64-token decode block
    and the 8192-token skewed block on the headline's packed GLM-5 expert weights
    (same shapes and distribution), and the GLM-4.7-Flash-shaped block on its own."""
    import torch

    from sigmoid_routed_mixture_b200 import moe

    out = {}
    for name in ("glm5_decode", "glm5_skewed", "glm47flash"):
        w = W.WORKLOADS[name]
        x, w_r, b = W.router_inputs(w)
        cfg = moe.Config.of(w)
        w_r_dev, b_dev = torch.from_numpy(w_r).to(dev), torch.from_numpy(b).to(dev)
        if name == "glm47flash":
            blk = moe.MoeBlock(cfg, w_r_dev, b_dev, **W.expert_weights(w, dev))
            weights_note = "its own seeded weights"
        else:
            blk = moe.MoeBlock(cfg, w_r_dev, b_dev, None, None, None, packed=packed)
            weights_note = "the headline block's packed GLM-5 expert weights (same shapes and distribution)"
        torch.cuda.empty_cache()
        x_dev = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
        step = build_step(cfg, blk, x_dev, False, stream)
        steps = steps_for(step, stream)
        meas = measure_block(step, blk.ws, steps, args.warmup, args.eager, None, stream)
        rec = {"value": w.T * steps / (meas["total_ms"] / 1e3), "unit": UNIT,
               "ms_per_step": meas["total_ms"] / steps, "steps": steps, "warmup": args.warmup,
               "tokens": w.T, "weights": weights_note,
               "launch": "cuda graph replay" if meas["graph"] is not None else "eager",
               "gpu_launches": kernels_per_step(w) * steps, "clocks": meas["clocks"]}
        rec.update(block_record(w, cfg, blk, meas, meas["total_ms"], steps, pk, False))
        out[name] = rec
        del meas, blk, step, x_dev
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="glm5_prefill",
                    choices=sorted(W.WORKLOADS) + sorted(W.DSA_WORKLOADS) + sorted(ROUTER_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=0)
    ap.add_argument("--cpu-tokens", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-also", action="store_true",
                    help="glm5_prefill at N = 1: skip timing the decode, skewed and GLM-4.7-Flash blocks")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--tokens", type=int, default=0, help="run the workload at this many tokens")
    ap.add_argument("--eager", action="store_true",
                    help="launch every step from the host instead of replaying a CUDA graph of it")
    ap.add_argument("--cublas", action="store_true",
                    help="dense workloads: also time torch.matmul (cuBLAS) on the same two GEMMs")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    is_dsa = args.workload in W.DSA_WORKLOADS
    if args.workload in ROUTER_WORKLOADS and args.impl == "reference":
        print(json.dumps({"impl": "reference", "unavailable": "the router stage bench has no oracle arm; the "
                          "block workloads time the oracle's router with the rest of the block"}), flush=True)
        return
    if args.impl == "reference":
        (run_dsa_reference if is_dsa else run_reference)(args, rank)
        return

    import torch

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    from sigmoid_routed_mixture_b200 import moe

    if args.workload in ROUTER_WORKLOADS:
        run_router(args, world, rank, dist, torch.device("cuda", torch.cuda.current_device()))
        if dist is not None:
            dist.destroy_process_group()
        return
    if is_dsa:
        run_dsa(args, world, rank, dist, torch.device("cuda", torch.cuda.current_device()))
        if dist is not None:
            dist.destroy_process_group()
        return
    w = W.WORKLOADS[args.workload]
    if args.tokens:
        w = w.replace(T=args.tokens)
    dev = torch.device("cuda", torch.cuda.current_device())
    # each replica draws its own token batch; weights are the workload's
    x, w_r, b = replica_tokens(w, rank)
    weights = W.expert_weights(w, dev)
    dense = w.E == 0
    cublas = None
    if dense:
        cfg = moe.Config.dense(w.T, w.H, w.I)
        blk = DenseBlock(cfg, moe.pack_weights(cfg, None, None, None, weights["ws1"], weights["ws3"],
                                               weights["ws2"]), dev)
        if args.cublas:  # the same two GEMMs through torch.matmul, for comparison only
            cublas = (torch.cat([weights["ws1"], weights["ws3"]], 0), weights["ws2"].clone(),
                      torch.randn((w.T, w.I), device=dev).to(torch.bfloat16))
    else:
        cfg = moe.Config.of(w)
        blk = moe.MoeBlock(cfg, torch.from_numpy(w_r).to(dev), torch.from_numpy(b).to(dev), **weights)
    del weights
    torch.cuda.empty_cache()
    x_dev = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    stream = torch.cuda.current_stream()
    step = build_step(cfg, blk, x_dev, dense, stream)
    meas = measure_block(step, blk.ws, args.steps, args.warmup, args.eager, dist, stream)
    graph = meas["graph"]
    total_ms = meas["total_ms"]
    t_max = max_over_ranks(total_ms, dist, dev)
    value = aggregate_tokens_per_s(w.T, world, args.steps, t_max)

    # ---- end to end: every step copies its token batch in from pinned host
    # memory and its output back to the host.  Two device buffer sets and
    # separate copy streams let step i + 1's input copy and step i - 1's output
    # copy run under step i's compute (the copies of every timed step are inside
    # the timed region).
    x_host = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    xs = [x_dev, torch.empty_like(x_dev)]
    ys = [blk.y, torch.empty_like(blk.y)]
    y_host = [torch.empty((w.T, w.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    replays = [graph.replay if graph is not None else (lambda: step(xin=xs[0], yout=ys[0]))]
    graph1 = None
    if graph is not None:
        step(xin=xs[1], yout=ys[1])
        torch.cuda.synchronize()
        graph1 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph1):
            step(xin=xs[1], yout=ys[1])
        replays.append(graph1.replay)
    else:
        replays.append(lambda: step(xin=xs[1], yout=ys[1]))
    e2e_ms = pipelined_e2e(torch, stream, dev, args.e2e_steps, dist,
                           lambda j: xs[j].copy_(x_host, non_blocking=True), replays,
                           lambda j: y_host[j].copy_(ys[j], non_blocking=True))
    e2e_value = aggregate_tokens_per_s(w.T, world, args.e2e_steps, e2e_ms)
    if moe.device_error(blk.ws) != 0:
        raise RuntimeError("device error during the timed steps")

    cublas_ms = None
    if cublas is not None:
        w13_t, w2_t, h_t = cublas

        def loop(fn):
            fn()
            torch.cuda.synchronize()
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(args.steps):
                fn()
            a1.record(stream)
            torch.cuda.synchronize()
            return a0.elapsed_time(a1) / args.steps

        cublas_ms = {"up": loop(lambda: torch.matmul(x_dev, w13_t.t())),
                     "down": loop(lambda: torch.matmul(h_t, w2_t.t()))}

    pk = peaks()
    rec = block_record(w, cfg, blk, meas, t_max, args.steps, pk, dense)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; random-init weights of the GLM-5 MoE block shapes)",
        "config": workload_config(w, argparse.Namespace(gpus=world)),
        "roofline": rec["roofline"],
        "block_roofline": rec["block_roofline"],
        "stage_ms": rec["stage_ms"],
        "launch": "cuda graph replay" if graph is not None else "eager",
        "eager_ms_per_step": meas["eager_ms"] / args.steps,
        "routing": rec["routing"],
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(w.T * w.H * 2),
                "d2h_bytes_per_step": int(w.T * w.H * 2), "steps": args.e2e_steps,
                "copies": "pinned host buffers, H2D and D2H on their own streams overlapping the compute of the "
                          "neighbouring steps (two device buffer sets)"},
        "gpu_launches": (KERNELS_PER_DENSE_STEP if dense else kernels_per_step(w)) * args.steps,
        "cublas_same_gemms_ms": cublas_ms,
        "clocks": meas["clocks"],
    }

    # ---- CPU baseline: the oracle on a bounded sample, rank 0 at N = 1 only
    if world == 1 and not args.no_cpu_baseline and not dense:
        os.environ.setdefault("OMP_NUM_THREADS", str(cores()))
        from oracle import oracle as O

        O.build()
        idx = blk.idx.cpu().numpy()
        n = args.cpu_tokens or max(8, min(2 * cores(), w.T))
        tokens = oracle_sample_tokens(w, idx, n)
        experts = set(np.unique(idx[tokens]).tolist())
        w13, w2p = blk.weights
        H, I = w.H, w.I

        def getter(name, e):
            # packed W13 of group e: units of 32 rows, 16 W1 rows then the matching 16 W3 rows
            if name in ("w1", "w3"):
                units = w13[e * 2 * I:(e + 1) * 2 * I].view(I // 16, 32, H)
                part = units[:, :16] if name == "w1" else units[:, 16:]
                return W.torch_bf16_to_bits(part.reshape(I, H))
            return W.torch_bf16_to_bits(w2p[e * H:(e + 1) * H].to(torch.bfloat16))

        tables = host_expert_tables(w, experts, getter)
        shared = [getter("w1", w.E), getter("w3", w.E), getter("w2", w.E)]
        # the same bounded sample repeated until the oracle has worked about 10 s
        # (at most ~30 s): more tokens would make the host hold more experts' weights
        times = run_oracle_steps(w, x, w_r, b, tokens, tables, shared, 1)
        while sum(times) < 10.0 and sum(times) + times[0] < 30.0:
            times += run_oracle_steps(w, x, w_r, b, tokens, tables, shared, 1)
        line["cpu_baseline"] = {
            "value": len(tokens) * len(times) / sum(times), "unit": UNIT,
            "cores": int(os.environ["OMP_NUM_THREADS"]), "kind": "oracle",
            "sample": "route+permute+forward of %d of the %d tokens, %d times (double-precision C oracle, "
                      "OpenMP), %.1f s" % (len(tokens), w.T, len(times), sum(times))}

    # ---- the other block configurations (after every timed region of the
    # headline, so they cannot disturb it), rank 0 at N = 1 only
    if world == 1 and not args.no_also and w.name == "glm5_prefill" and not args.tokens:
        packed = blk.weights
        del replays, graph, graph1, meas, step
        line["also"] = also_records(args, dev, stream, pk, packed)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
