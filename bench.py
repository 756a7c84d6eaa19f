"""Benchmark of the GALE 1-bit MoE expert layer on B200.

Workload: one routed-expert MoE layer at decode batch 1 -- 256 GALE-1bit
SwiGLU experts, w1/w3 [2048 x 4096], w2 [4096 x 2048] (about 1.07 GB packed,
all resident), top-6 routing with gates softmax-normalised over the selected
six, bf16 hidden states N(0,1) [1 x 4096].  A step is one gale_moe_forward
call: routing permute, FWHT of x, fused w1/w3 GEMV + SwiGLU, FWHT of h, w2
GEMV, gate-weighted combine.  Every step uses a fresh routing from a seeded
pool, and L2 is flushed (a write larger than L2) between timed steps, outside
the timed events.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
For N > 1 launch under torch.distributed.run: every rank runs its own replica
(weak scaling, no collective on the data path); rank 0 prints one JSON line.
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

import gale_synth as gs  # noqa: E402

METRIC = "MoE expert-layer tokens/s and packed-expert HBM GB/s (% of B200 roofline)"
UNIT = "tokens/s"
D_MODEL, D_FF, N_EXPERTS, TOP_K = 4096, 2048, 256, 6
PREFILL_B = 4096
CHAIN_LAYERS = 43
# rows of the 4-bit non-expert GEMV line (x d_model columns: 138 MB of 4-bit weights)
W4_ROWS = 65536
# kernels of this library launched per decode step (the cooperative layer kernel)
DECODE_LAUNCHES = 1
# dram read + write bytes of one decode launch at this workload, from an ncu
# capture (profiles/moe_decode_kernel_b1.md), and the sha256 prefix of the
# kernel source it was taken on: the bench reports it only while the source is
# unchanged, and null after any edit until the capture is taken again.
DECODE_TRAFFIC = 25_199_104
DECODE_TRAFFIC_SRC = "212e84e48af81dae"
KERNEL_SRC = os.path.join(ROOT, "bit_expert_gemv_b200", "csrc", "moe_decode.cu")


def decode_traffic():
    import hashlib
    if DECODE_TRAFFIC is None:
        return None
    with open(KERNEL_SRC, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()[:16]
    return DECODE_TRAFFIC if h == DECODE_TRAFFIC_SRC else None
WORKLOAD = ("moe_layer_decode: 256 GALE-1bit experts (w1/w3 [2048x4096], w2 [4096x2048]), "
            "top-6 softmax routing, bf16 hidden [B x 4096]")


def peaks():
    """HBM GB/s and dense 16-bit tensor TFLOP/s (burst) of this machine's B200s."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def relaunch_replicas(n: int):
    """`bench.py --gpus N` started without torchrun: run the same command as N
    replica processes under torch.distributed.run (one per GPU)."""
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    os.execv(sys.executable, cmd)


def max_over_ranks(values, world, device):
    """Per-rank device times -> their maximum over all ranks (every rank gets
    it).  One all-reduce, the same on every rank, whatever the backend."""
    import torch
    import torch.distributed as dist
    tt = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return [float(v) for v in tt.tolist()]


def job_throughput(batch, steps, world, t_max):
    """Whole-job tokens and tokens/s: every rank is an independent replica
    running `steps` steps of `batch` tokens; the job takes the slowest
    rank's time."""
    tokens = batch * steps * world
    return tokens, tokens / t_max


# ----------------------------------------------------------------------------
# clocks sampling (nvidia-smi during the timed region)
# ----------------------------------------------------------------------------

class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(os.environ.get("GALE_CLOCKS_DIR", tempfile.gettempdir()),
                                 f"gale_clocks_rank{index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader",
                                          "-i", str(self.index), "-lms", "50"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # the sampler takes a moment to start: the timed region begins after its first line
        t0 = time.time()
        while time.time() - t0 < 10.0 and self.proc.poll() is None:
            self.fh.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1].split()[0]))
                    smax.append(float(parts[2].split()[0]))
                except ValueError:
                    continue
                for n, v in zip(names[1:], parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# the layer on the device
# ----------------------------------------------------------------------------

def build_layer(torch, G, layer_id: int = 0, dst=None):
    """Pack 256 seeded experts into one resident device buffer: the seeded
    canonical matrices are drawn on the device (torch port of the generator)
    and packed by gale_pack."""
    stride = G.gale_expert_bytes(D_MODEL, D_FF)
    buf = dst if dst is not None else torch.empty(N_EXPERTS * stride, dtype=torch.uint8, device="cuda")
    l1 = G.gale_pack_layout(D_FF, D_MODEL)["total"]
    offs = [0, l1, 2 * l1]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    shapes = [(D_FF, D_MODEL, gs.W1), (D_FF, D_MODEL, gs.W3), (D_MODEL, D_FF, gs.W2)]
    chunk = 16
    for m, (rows, cols, mat) in enumerate(shapes):
        for e0 in range(0, N_EXPERTS, chunk):
            es = list(range(e0, min(N_EXPERTS, e0 + chunk)))
            c = gs.matrices_canonical_torch(rows, cols, layer_id, es, mat, device="cuda")
            for i, e in enumerate(es):
                G.gale_pack(c["signs"][i], c["s_blk"][i], c["s_row"][i], c["idx"][i], c["q"][i], rows, cols,
                            buf[e * stride + offs[m]:], status)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError("gale_pack reported invalid outliers")
    return buf, stride


def routing_pool(n: int, B: int, tag0: int, bias_sigma: float = 0.0, n_x: int = 0):
    """n seeded (hidden, ids, gates, distinct experts) steps; n_x > 0 reuses
    that many hidden-state draws (large batches: the routing is what varies)."""
    pool = []
    xs = [gs.hidden_bf16(B, D_MODEL, tag=tag0 + i)[0] for i in range(n_x)] if n_x else None
    for i in range(n):
        lg = gs.router_logits(B, N_EXPERTS, tag=tag0 + i, bias_sigma=bias_sigma)
        ids, gates = gs.route_topk(lg, TOP_K)
        bits = xs[i % n_x] if n_x else gs.hidden_bf16(B, D_MODEL, tag=tag0 + i)[0]
        pool.append((bits, ids, gates, len(np.unique(ids))))
    return pool


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import bit_expert_gemv_b200 as G

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=300))
    G.lib()
    buf, stride = build_layer(torch, G)
    layer = G.make_layer(buf, stride, N_EXPERTS, D_MODEL, D_FF)
    expert_bytes = stride
    l2 = torch.cuda.get_device_properties(local).L2_cache_size if hasattr(
        torch.cuda.get_device_properties(local), "L2_cache_size") else 126 * 2 ** 20
    flush = torch.empty(max(2 * l2, 256 * 2 ** 20), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def measure(B, steps, warmup, tag0, bias_sigma=0.0, n_x=0):
        pool = routing_pool(steps + warmup, B, tag0 + 7919 * rank, bias_sigma, n_x)
        dev = [(torch.from_numpy(b).view(torch.bfloat16).cuda(), torch.from_numpy(i).cuda(),
                torch.from_numpy(g).cuda(), nd) for b, i, g, nd in pool]
        ws = torch.empty(G.gale_moe_workspace_size(layer, B, TOP_K), dtype=torch.uint8, device="cuda")
        out = torch.empty(B, D_MODEL, dtype=torch.float32, device="cuda")
        for s in range(warmup):
            x, ids, gates, _ = dev[s]
            G.gale_moe_forward(layer, x, ids, gates, out, ws)
        torch.cuda.synchronize()
        if int(ws[:4].view(torch.int32).item()) != 0:
            raise RuntimeError("device status after warm-up")
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for s in range(steps):
            x, ids, gates, _ = dev[warmup + s]
            flush.zero_()
            ev[s][0].record(stream)
            G.gale_moe_forward(layer, x, ids, gates, out, ws)
            ev[s][1].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        times = [a.elapsed_time(b) * 1e-3 for a, b in ev]
        total = sum(times)
        n_bytes = sum(dev[warmup + s][3] for s in range(steps)) * expert_bytes
        return total, n_bytes, times

    def measure_e2e(B, steps, warmup, tag0):
        """Through the public host-buffer call (gale_moe_forward_host): the
        inputs in pinned host memory cross in one packed copy, the layer
        runs, and the result lands in pinned host memory, every step."""
        pool = routing_pool(steps + warmup, B, tag0 + 7919 * rank)
        host = [(torch.from_numpy(b).view(torch.bfloat16).pin_memory(), torch.from_numpy(i).pin_memory(),
                 torch.from_numpy(g).pin_memory()) for b, i, g, _ in pool]
        staging = torch.empty(G.gale_moe_host_staging_bytes(B, TOP_K, D_MODEL), dtype=torch.uint8).pin_memory()
        ws = torch.empty(G.gale_moe_host_workspace_size(layer, B, TOP_K), dtype=torch.uint8, device="cuda")
        out_h = torch.empty(B, D_MODEL, dtype=torch.float32).pin_memory()

        def step(s):
            x, i, g = host[s]
            G.gale_moe_forward_host(layer, x, i, g, out_h, ws, staging)

        for s in range(warmup):
            step(s)
            torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for s in range(steps):
            flush.zero_()
            ev[s][0].record(stream)
            step(warmup + s)
            ev[s][1].record(stream)
            torch.cuda.synchronize()   # the result is in host memory; staging may be refilled
        total = sum(a.elapsed_time(b) * 1e-3 for a, b in ev)
        h2d = staging.numel()
        d2h = B * D_MODEL * 4
        return total, h2d, d2h

    def measure_single(steps, warmup):
        """One GALE expert on one token, x fp32 N(0,1) [4096]: FWHT of x, the
        fused w1/w3 GEMV + SwiGLU, FWHT of h, the w2 GEMV (expert 0 of the
        resident layer), L2 flushed before every step (outside the events)."""
        l1 = G.gale_pack_layout(D_FF, D_MODEL)["total"]
        w1, w3, w2 = buf[0:], buf[l1:], buf[2 * l1:]
        xs = [torch.from_numpy(gs.x_f32(D_MODEL, tag=95_000 + i)).cuda().view(1, D_MODEL)
              for i in range(steps + warmup)]
        xr = torch.empty(1, D_MODEL, dtype=torch.float32, device="cuda")
        h = torch.empty(1, D_FF, dtype=torch.float32, device="cuda")
        y = torch.empty(1, D_MODEL, dtype=torch.float32, device="cuda")

        def step(x):
            G.gale_fwht1024(x, xr)
            G.gale_expert_gemv(w1, D_FF, D_MODEL, xr, h, W3=w3, mode=G.GALE_MODE_SWIGLU)
            G.gale_fwht1024(h, h)
            G.gale_expert_gemv(w2, D_MODEL, D_FF, h, y)

        wsf = torch.empty(G.gale_expert_forward_workspace_size(layer, 1), dtype=torch.uint8, device="cuda")

        def fused(x):
            G.gale_expert_forward(layer, 0, x, y, wsf)

        times = []
        for fn in (step, fused):
            for i in range(warmup):
                fn(xs[i])
            torch.cuda.synchronize()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for i in range(steps):
                flush.zero_()
                ev[i][0].record(stream)
                fn(xs[warmup + i])
                ev[i][1].record(stream)
            torch.cuda.synchronize()
            times.append(sum(a.elapsed_time(b) * 1e-3 for a, b in ev))
        return times[0], times[1]

    def measure_w4(steps, warmup, B):
        """The 4-bit non-expert weight GEMV (symmetric int4, 128-block fp16
        scales): one [W4_ROWS x D_MODEL] matrix quantized on the device from
        seeded N(0, 0.02) weights, B bf16 tokens, L2 flushed before every
        step (outside the events).  Returns (seconds, bytes per step)."""
        L = G.gale_w4_layout(W4_ROWS, D_MODEL)
        packed = torch.empty(L.total, dtype=torch.uint8, device="cuda")
        key = gs.stream_key(73, 0)
        w = torch.empty(W4_ROWS, D_MODEL, dtype=torch.float32, device="cuda")
        rows_per = 4096
        for r0 in range(0, W4_ROWS, rows_per):   # drawn in slices of rows
            w[r0:r0 + rows_per] = (gs.normal_torch(key, rows_per * D_MODEL, start=r0 * D_MODEL) * 0.02).view(
                rows_per, D_MODEL)
        G.gale_w4_quantize(w, packed)
        del w
        xs = [torch.from_numpy(gs.hidden_bf16(B, D_MODEL, tag=97_000 + i)[0]).view(torch.int16).cuda()
              for i in range(steps + warmup)]
        y = torch.empty(B, W4_ROWS, dtype=torch.float32, device="cuda")
        ws = torch.zeros(G.gale_w4_workspace_size(W4_ROWS, D_MODEL, B), dtype=torch.uint8, device="cuda")
        for i in range(warmup):
            G.gale_w4_gemv(packed, W4_ROWS, D_MODEL, xs[i], y, ws)
        torch.cuda.synchronize()
        if int(ws[:4].view(torch.int32).item()) != 0:
            raise RuntimeError("4-bit GEMV status after warm-up")
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.zero_()
            ev[i][0].record(stream)
            G.gale_w4_gemv(packed, W4_ROWS, D_MODEL, xs[warmup + i], y, ws)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        t = sum(a.elapsed_time(b) * 1e-3 for a, b in ev)
        return t, L.total + B * D_MODEL * 2 + B * W4_ROWS * 4

    def measure_chain(steps, warmup, n_layers=CHAIN_LAYERS):
        """Decode batch 1 through n_layers layers of 256 resident experts each:
        x_{l+1} = bf16(RMSNorm(x_l + MoE_l(x_l))), fresh seeded routing per
        layer and step.  46 GB of packs are far larger than L2, so every layer
        reads its experts from HBM.  Returns (seconds, packed bytes read, used graph)."""
        lb = N_EXPERTS * expert_bytes
        big = torch.empty(n_layers * lb, dtype=torch.uint8, device="cuda")
        layers = []
        for l in range(n_layers):
            build_layer(torch, G, layer_id=l, dst=big[l * lb:(l + 1) * lb])
            layers.append(G.make_layer(big[l * lb:], expert_bytes, N_EXPERTS, D_MODEL, D_FF))
        n = steps + warmup
        # per-layer router logits N(0,1) over the 256 experts; the graph routes on
        # the device (top-6, softmax over the six) before every layer
        logits = torch.empty(n, n_layers, 1, N_EXPERTS, dtype=torch.float32, device="cuda")
        distinct = 0
        for s in range(n):
            for l in range(n_layers):
                lg = gs.router_logits(1, N_EXPERTS, tag=90_000 + 1000 * s + l)
                logits[s, l] = torch.from_numpy(lg)
                if s >= warmup:
                    distinct += len(np.unique(gs.route_topk(lg, TOP_K)[0]))
        x0 = torch.from_numpy(gs.hidden_bf16(1, D_MODEL, tag=91_000)[0]).view(torch.bfloat16).cuda()
        ws = torch.empty(G.gale_moe_workspace_size(layers[0], 1, TOP_K), dtype=torch.uint8, device="cuda")
        xb = [torch.empty(1, D_MODEL, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        cur_lg = torch.empty(n_layers, 1, N_EXPERTS, dtype=torch.float32, device="cuda")
        cur_ids = torch.empty(n_layers, 1, TOP_K, dtype=torch.int32, device="cuda")
        cur_g = torch.empty(n_layers, 1, TOP_K, dtype=torch.float32, device="cuda")

        def token():
            x = x0
            for l in range(n_layers):
                G.gale_route_topk(cur_lg[l], cur_ids[l], cur_g[l])
                G.gale_moe_forward(layers[l], x, cur_ids[l], cur_g[l], xb[l % 2], ws,
                                   flags=G.GALE_FLAG_RESIDUAL_RMSNORM, eps=1e-6)
                x = xb[l % 2]

        for s in range(warmup):
            cur_lg.copy_(logits[s])
            token()
        torch.cuda.synchronize()
        if int(ws[:4].view(torch.int32).item()) != 0:
            raise RuntimeError("device status after chain warm-up")
        graph = None
        try:   # the 43 launches of a token as one CUDA graph
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                token()
            graph = g
        except Exception:
            graph = None
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for s in range(steps):
            cur_lg.copy_(logits[warmup + s])
            ev[s][0].record(stream)
            if graph is not None:
                graph.replay()
            else:
                token()
            ev[s][1].record(stream)
        torch.cuda.synchronize()
        t = sum(a.elapsed_time(b) * 1e-3 for a, b in ev)
        # the same stack as one persistent launch (gale_moe_chain) after one
        # router launch for every layer: two launches per token
        first = layers[0]
        wsc = torch.empty(G.gale_moe_chain_workspace_size(first, n_layers, 1, TOP_K), dtype=torch.uint8,
                          device="cuda")
        xo = torch.empty(1, D_MODEL, dtype=torch.bfloat16, device="cuda")
        lg2 = cur_lg.view(n_layers, N_EXPERTS)
        ids2 = cur_ids.view(n_layers, TOP_K)
        g2 = cur_g.view(n_layers, TOP_K)

        def token_chain():
            G.gale_route_topk(lg2, ids2, g2)
            G.gale_moe_chain(first, n_layers, lb, x0, cur_ids, cur_g, xo, wsc)

        for s in range(warmup):
            cur_lg.copy_(logits[s])
            token_chain()
        torch.cuda.synchronize()
        if int(wsc[:4].view(torch.int32).item()) != 0:
            raise RuntimeError("device status after persistent chain warm-up")
        evc = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for s in range(steps):
            cur_lg.copy_(logits[warmup + s])
            evc[s][0].record(stream)
            token_chain()
            evc[s][1].record(stream)
        torch.cuda.synchronize()
        tk = sum(a.elapsed_time(b) * 1e-3 for a, b in evc)
        del big
        torch.cuda.empty_cache()
        return t, distinct * expert_bytes, graph is not None, tk

    # nvidia-smi samples the clocks through every timed measurement below
    clocks = Clocks(local)
    clocks.start()
    t1, bytes1, times1 = measure(1, args.steps, args.warmup, 10_000)
    t8, bytes8, _ = measure(8, max(args.steps // 2, 3), args.warmup, 20_000)
    # decode batch 64 with per-expert popularity bias N(0, 0.5) (skewed tokens per expert)
    t64, bytes64, _ = measure(64, max(args.steps // 2, 3), args.warmup, 25_000, bias_sigma=0.5)
    te, h2d, d2h = measure_e2e(1, args.steps, args.warmup, 30_000)
    ts, tsf = measure_single(args.steps, args.warmup)
    tw1, w4b1 = measure_w4(args.steps, args.warmup, 1)
    tw8, w4b8 = measure_w4(args.steps, args.warmup, 8)
    # prefill: 4096 tokens, skewed routing (tensor-core tile path)
    pf_steps = max(3, min(args.steps // 5, 10))
    tp, _, _ = measure(PREFILL_B, pf_steps, 3, 40_000, bias_sigma=0.5, n_x=2)
    ch_steps = max(3, min(args.steps // 5, 10))
    tc, bytes_c, ch_graph, tck = measure_chain(ch_steps, 3) if not args.no_chain else (float("nan"), 0, False,
                                                                                         float("nan"))
    clocks_info = clocks.stop()

    # max over ranks of the device time
    t1, t8, t64, te, tp, tc, ts, tw1, tw8, tck, tsf = max_over_ranks([t1, t8, t64, te, tp, tc, ts, tw1, tw8, tck, tsf],
                                                                      world, "cuda")
    tokens, value = job_throughput(1, args.steps, world, t1)
    gbs = bytes1 * world / t1 / 1e9
    peak, tpeak, peak_kind = peaks()
    pf_flops = 2.0 * PREFILL_B * TOP_K * 3 * D_FF * D_MODEL   # dense-equivalent, per layer
    avg_launch = t1 / args.steps
    achieved = bytes1 / args.steps / avg_launch / 1e9
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * t1 / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "s8x3 fixed-point activations x 1-bit signs, s32 accumulate, fp32 scales and sums",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": 1, "experts": N_EXPERTS, "top_k": TOP_K,
                   "d_model": D_MODEL, "d_ff": D_FF, "packed_bytes_per_expert": expert_bytes,
                   "l2": "flushed between timed steps (write of 2x L2, outside the events)",
                   "routing": "fresh seeded routing every step", "parallelism": f"replicas{world}"},
        "hbm_gbs": gbs,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": decode_traffic(), "peak_kind": peak_kind,
                     "kernel": "moe_decode_kernel (batch 1: the whole layer is this one launch)",
                     "algorithmic_bytes_per_launch": bytes1 / args.steps},
        "b8": {"tokens_per_s": 8 * max(args.steps // 2, 3) * world / t8,
               "hbm_gbs": bytes8 * world / t8 / 1e9, "frac": bytes8 * world / t8 / 1e9 / peak},
        "b64": {"tokens_per_s": 64 * max(args.steps // 2, 3) * world / t64,
                "ms_per_step": 1e3 * t64 / max(args.steps // 2, 3),
                "hbm_gbs": bytes64 * world / t64 / 1e9, "frac": bytes64 * world / t64 / 1e9 / peak,
                "routing": "top-6 with per-expert bias N(0, 0.5) (skewed)"},
        "chain43": {"workload": f"decode batch 1 through {CHAIN_LAYERS} layers x 256 resident experts "
                                f"(46 GB), router on the device (top-6 of per-layer logits), residual + RMSNorm "
                                f"between layers, bf16 hidden state",
                    "tokens_per_s": ch_steps * world / tc, "ms_per_token": 1e3 * tc / ch_steps,
                    "hbm_gbs": bytes_c * world / tc / 1e9, "frac": bytes_c * world / tc / 1e9 / peak,
                    "cuda_graph": ch_graph, "steps": ch_steps,
                    "persistent": {"launches_per_token": 2,
                                   "what": "one router launch for all layers, then gale_moe_chain (one cooperative "
                                           "launch for the 43 layers)",
                                   "tokens_per_s": ch_steps * world / tck, "ms_per_token": 1e3 * tck / ch_steps,
                                   "hbm_gbs": bytes_c * world / tck / 1e9,
                                   "frac": bytes_c * world / tck / 1e9 / peak}},
        "prefill": {"workload": "4096 tokens, top-6 with per-expert bias N(0, 0.5) (skewed), same 256 experts",
                    "tokens_per_s": PREFILL_B * pf_steps * world / tp, "ms_per_step": 1e3 * tp / pf_steps,
                    "tflops": pf_flops * pf_steps / tp / 1e12, "peak_tflops": tpeak,
                    "frac": pf_flops * pf_steps / tp / 1e12 / tpeak, "bound": "tensor",
                    "flops_per_step": pf_flops, "steps": pf_steps},
        "single_expert": {"workload": "one GALE expert, one token, fp32 x [4096] (w1/w3 [2048x4096], w2 [4096x2048]), "
                                      "L2 flushed: gale_expert_forward (one launch)",
                          "tokens_per_s": args.steps * world / tsf, "us_per_step": 1e6 * tsf / args.steps,
                          "hbm_gbs": expert_bytes * args.steps * world / tsf / 1e9,
                          "frac": expert_bytes * args.steps * world / tsf / 1e9 / peak, "launches_per_step": 1,
                          "four_launches": {"what": "FWHT, w1/w3 GEMV + SwiGLU, FWHT, w2 GEMV (gale_fwht1024, "
                                                    "gale_expert_gemv)",
                                            "us_per_step": 1e6 * ts / args.steps,
                                            "frac": expert_bytes * args.steps * world / ts / 1e9 / peak}},
        "w4_gemv": {"workload": f"4-bit non-expert weight GEMV: symmetric int4, fp16 scale per 128-block, "
                                f"[{W4_ROWS} x {D_MODEL}] (quantized on the device from seeded N(0, 0.02)), "
                                f"bf16 tokens, L2 flushed (one launch)",
                    "b1": {"us_per_step": 1e6 * tw1 / args.steps, "hbm_gbs": w4b1 * args.steps * world / tw1 / 1e9,
                           "frac": w4b1 * args.steps * world / tw1 / 1e9 / peak, "bytes_per_step": w4b1},
                    "b8": {"us_per_step": 1e6 * tw8 / args.steps, "hbm_gbs": w4b8 * args.steps * world / tw8 / 1e9,
                           "frac": w4b8 * args.steps * world / tw8 / 1e9 / peak, "bytes_per_step": w4b8},
                    "bound": "hbm"},
        "e2e": {"value": tokens / te, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": DECODE_LAUNCHES * args.steps,
        "clocks": clocks_info,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def run_profile_w4(args):
    """ncu driver of the 4-bit GEMV: the [W4_ROWS x D_MODEL] matrix of the bench
    line, --warmup calls, an L2 flush, then --steps calls with --batch tokens."""
    import torch
    import bit_expert_gemv_b200 as G
    G.lib()
    B = args.batch
    L = G.gale_w4_layout(W4_ROWS, D_MODEL)
    packed = torch.empty(L.total, dtype=torch.uint8, device="cuda")
    w = torch.empty(W4_ROWS, D_MODEL, dtype=torch.float32, device="cuda")
    for r0 in range(0, W4_ROWS, 4096):
        w[r0:r0 + 4096] = (gs.normal_torch(gs.stream_key(73, 0), 4096 * D_MODEL, start=r0 * D_MODEL) * 0.02).view(
            4096, D_MODEL)
    G.gale_w4_quantize(w, packed)
    del w
    x = torch.from_numpy(gs.hidden_bf16(B, D_MODEL, tag=97_000)[0]).view(torch.int16).cuda()
    y = torch.empty(B, W4_ROWS, dtype=torch.float32, device="cuda")
    ws = torch.zeros(G.gale_w4_workspace_size(W4_ROWS, D_MODEL, B), dtype=torch.uint8, device="cuda")
    flush = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        G.gale_w4_gemv(packed, W4_ROWS, D_MODEL, x, y, ws)
    torch.cuda.synchronize()
    flush.zero_()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        G.gale_w4_gemv(packed, W4_ROWS, D_MODEL, x, y, ws)
    torch.cuda.synchronize()
    print(json.dumps({"profile": "w4", "batch": B, "steps": args.steps}), flush=True)


def run_profile(args):
    """A short fixed sequence for ncu captures: build the layer, run
    --warmup calls, flush L2, run --steps calls (decode: unbiased routing;
    prefill: per-expert bias N(0, 0.5)), print the device status."""
    import torch
    import bit_expert_gemv_b200 as G
    if args.only == "w4":
        return run_profile_w4(args)
    G.lib()
    buf, stride = build_layer(torch, G)
    layer = G.make_layer(buf, stride, N_EXPERTS, D_MODEL, D_FF)
    B = args.batch
    pool = routing_pool(args.steps + args.warmup, B, 80_000, 0.5 if args.only == "prefill" else 0.0,
                        n_x=2 if B > 64 else 0)
    dev = [(torch.from_numpy(b).view(torch.bfloat16).cuda(), torch.from_numpy(i).cuda(),
            torch.from_numpy(g).cuda()) for b, i, g, _ in pool]
    ws = torch.empty(G.gale_moe_workspace_size(layer, B, TOP_K), dtype=torch.uint8, device="cuda")
    out = torch.empty(B, D_MODEL, dtype=torch.float32, device="cuda")
    flush = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device="cuda")
    for s in range(args.warmup):
        G.gale_moe_forward(layer, *dev[s], out, ws)
    torch.cuda.synchronize()
    flush.zero_()
    torch.cuda.synchronize()
    for s in range(args.steps):
        G.gale_moe_forward(layer, *dev[args.warmup + s], out, ws)
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.only, "batch": B, "steps": args.steps,
                      "status": int(ws[:4].view(torch.int32).item())}), flush=True)


# ----------------------------------------------------------------------------
# CPU oracle timings
# ----------------------------------------------------------------------------

def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_inputs(O, n: int, tag0: int):
    """n decode-batch-1 steps of seeded routing and hidden states, with every
    expert they touch generated and packed by the oracle's own packer; all of
    this happens before any timing."""
    steps = []
    for i in range(n):
        ids, gates = gs.route_topk(gs.router_logits(1, N_EXPERTS, tag=tag0 + i), TOP_K)
        _, xv = gs.hidden_bf16(1, D_MODEL, tag=tag0 + i)
        packed = {int(e): [O.pack(c) for c in gs.expert_canonical(D_MODEL, D_FF, expert=int(e))]
                  for e in np.unique(ids)}
        steps.append((xv, ids, gates, packed))
    return steps


def oracle_step(O, step):
    """The oracle on one prepared step: unpack and dense fp64 dequantisation
    of the six experts, FWHT, SwiGLU, w2 and the gate-weighted combine."""
    xv, ids, gates, packed = step
    shapes = [(D_FF, D_MODEL), (D_FF, D_MODEL), (D_MODEL, D_FF)]
    dense = {e: [O.dequant_packed(b, r, c) for b, (r, c) in zip(v, shapes)] for e, v in packed.items()}
    O.moe_layer(dense.__getitem__, xv, ids, gates)
    return 1


def cpu_baseline(budget_s: float):
    """The oracle as it stands on the host cores: half the budget on all BLAS
    threads, half on one thread (experts generated and packed beforehand)."""
    from oracle import gale_oracle as O
    from threadpoolctl import threadpool_limits
    inputs = oracle_inputs(O, 8, 50_000)
    oracle_step(O, inputs[0])   # first touch of the allocator's pages, untimed
    res = {}
    for label, limit in (("all", None), ("one", 1)):
        ctx = threadpool_limits(limit) if limit else None
        if ctx:
            ctx.__enter__()
        try:
            cores = _threads()
            t0 = time.perf_counter()
            n = 0
            while (time.perf_counter() - t0 < budget_s / 2 or n == 0) and n < len(inputs):
                oracle_step(O, inputs[(n + 1) % len(inputs)])
                n += 1
            res[label] = (n / (time.perf_counter() - t0), cores, n)
        finally:
            if ctx:
                ctx.__exit__(None, None, None)
    v, cores, n = res["all"]
    v1, _, n1 = res["one"]
    return {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} decode-B1 layer steps on {cores} threads and {n1} on one (6 experts each: unpack, "
                      f"dense fp64 dequant, FWHT, SwiGLU, w2, combine; experts packed before the clock)",
            "single_thread": {"value": v1, "unit": UNIT, "cores": 1}}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from oracle import gale_oracle as O
    inputs = oracle_inputs(O, min(args.steps, 8), 70_000)
    for s in range(args.warmup):
        oracle_step(O, inputs[s % len(inputs)])
    t0 = time.perf_counter()
    for s in range(args.steps):
        oracle_step(O, inputs[s % len(inputs)])
    dt = time.perf_counter() - t0
    value = args.steps / dt
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": 1, "experts": N_EXPERTS, "top_k": TOP_K},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _threads(), "kind": "oracle",
                         "sample": f"{args.steps} decode-B1 layer steps (experts packed before the clock)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="gale", choices=["gale", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-chain", action="store_true", help="skip the 43-layer chain measurement")
    ap.add_argument("--only", choices=["decode", "prefill", "w4"], default=None,
                    help="profiling driver: warm-up, an L2 flush, then --steps layer calls of one path")
    ap.add_argument("--batch", type=int, default=1, help="tokens per step with --only")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        relaunch_replicas(args.gpus)
    if args.impl == "reference":
        run_reference(args)
    elif args.only:
        run_profile(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
