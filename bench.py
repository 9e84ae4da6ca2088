#!/usr/bin/env python
"""ReSA decode hot-path benchmark on B200.

One step = one ReSA cycle of f = 32 tokens through every layer: f-1 sparse
decode steps (append + block selection + group block-sparse split-KV
attention) followed by one dense rectification of the last f tokens
(write-back + descriptor refresh + causal chunk attention), per layer, as in
Algorithm 1 of the Rectified Sparse Attention summary.  Each cycle is one CUDA
graph of libresa launches; inputs are seeded synthetic tensors resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long256k]
    python bench.py --impl reference ...     # the CPU oracle on the same workload

Multi-GPU: one process per GPU (torchrun); the path does not shard, so every
rank runs an independent replica (weak scaling) and the time is the maximum
over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-decode attn tokens/s & µs/step at 256K ctx; achieved HBM GB/s vs B200 peak"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

WORKLOADS = {
    "long256k": dict(layers=28, batch=1, hq=28, hkv=4, d=128, ctx=[262144], f=32, paged=False,
                     text="long-context decode: 28 layers x (28 q / 4 kv heads, d 128), batch 1, "
                          "262144-token bf16 cache, block 16, top-k 10% (1638) + current block, "
                          "ReSA cycle f=32 (31 sparse decode steps + 1 dense rectification)"),
    "layer256k": dict(layers=1, batch=1, hq=28, hkv=4, d=128, ctx=[262144], f=32, paged=False,
                      text="one layer of the long-context decode workload (28 q / 4 kv, d 128), "
                           "262144-token cache, top-k 10% + current block, ReSA cycle f=32"),
    "qwen32k": dict(layers=4, batch=1, hq=28, hkv=4, d=128, ctx=[32768], f=32, paged=False,
                    text="one attention layer of Qwen2.5-7B shape (28 q / 4 kv, d 128), batch 1, "
                         "32768-token cache, top-k 10% (205) + current block; timed over 4 "
                         "independent layer caches in turn (268 MB) so that L2 cannot hold "
                         "the cache, reported per layer"),
    "loop64k": dict(layers=1, batch=4, hq=28, hkv=4, d=128, ctx=[65536] * 4, f=32, paged=False,
                    text="ReSA decode loop: 1 layer (28 q / 4 kv, d 128), batch 4, 65536-token "
                         "cache, top-k 10%, 31 sparse decode steps + 1 rectification of 32"),
    "cbatch": dict(layers=1, batch=32, hq=28, hkv=4, d=128, ctx=None, f=32, paged=True,
                   text="continuous batching: 1 layer, 32 sequences with lengths uniform in "
                        "[8192, 131072], random page order, top-k 10% per sequence"),
    "tiny": dict(layers=1, batch=1, hq=4, hkv=2, d=64, ctx=[2048], f=32, paged=False,
                 text="tiny: 1 layer (4 q / 2 kv, d 64), 2048-token cache, top-k 16"),
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["resa", "reference"], default="resa")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="long256k")
    ap.add_argument("--seed", type=int, default=1234)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the dense baseline and the further workloads")
    ap.add_argument("--breakdown-reps", type=int, default=5)
    ap.add_argument("--sweep-block-sizes", default="16,32,64",
                    help="block sizes b of --sweep (comma-separated)")
    ap.add_argument("--sweep", action="store_true",
                    help="time the decode step over top-k fractions and the rectification over "
                         "chunk lengths f, and compare the per-token cost with Eq. 6 (prints one "
                         "JSON line, not the benchmark line)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# Distributed plumbing (replicas only: no collective on the data path)
# ---------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_setup(backend: str, world: int):
    if world <= 1:
        return None
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
    return dist


def max_over_ranks(x: float, dist=None, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity with one rank)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist=None, device=None):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# Workload construction
# ---------------------------------------------------------------------------

def bench_config(name, wl):
    """The workload description both arms print (the same dict)."""
    return {"workload": name, "description": wl["text"],
            "step": f"one ReSA cycle of {wl['f']} tokens through {wl['layers']} layers",
            "l2": "working set larger than L2 (cache > 126 MB per layer set); no flush",
            "parallelism": "replicas, one per GPU, no data-path collective"}


def topk_rule(L: int, bs: int = 16, n_min: int = 16) -> int:
    """top-k of a decode step: max(n_min, round(M / 10)) capped at M, M = (L-1)//bs."""
    M = (L - 1) // bs
    return min(M, max(n_min, (M + 5) // 10))


def workload_lengths(wl, seed):
    from block_sparse_long_resa_b200 import inputs
    if wl["ctx"] is None:
        return inputs.continuous_batch_lengths(seed, wl["batch"], 8192, 131072)
    return list(wl["ctx"])


class Schedule:
    """Sequence lengths and top-k per global step (decode steps and rectifications)."""

    def __init__(self, ctx, f, cycles, bs=16):
        self.ctx, self.f, self.cycles, self.bs = ctx, f, cycles, bs
        self.B = len(ctx)
        self.Bpad = (self.B + 3) // 4 * 4  # 16-byte aligned rows

    def decode_L(self, c, s):
        return [L0 + c * self.f + s + 1 for L0 in self.ctx]

    def rect_L(self, c):
        return [L0 + (c + 1) * self.f for L0 in self.ctx]

    def max_topk(self):
        return max(topk_rule(L0 + self.cycles * self.f, self.bs) for L0 in self.ctx)

    def total_tokens(self):
        return max(self.ctx) + self.cycles * self.f


class GpuWorkload:
    def __init__(self, wl, cycles, seed, device, bs=16):
        import torch
        from block_sparse_long_resa_b200 import inputs
        from block_sparse_long_resa_b200 import resa as R
        self.wl, self.dev, self.cycles = wl, device, cycles
        self.R = R
        B, hq, hkv, d, f, nl = wl["batch"], wl["hq"], wl["hkv"], wl["d"], wl["f"], wl["layers"]
        self.B, self.hq, self.hkv, self.d, self.f, self.layers = B, hq, hkv, d, f, nl
        self.bs = bs
        ctx = workload_lengths(wl, seed)
        self.sched = Schedule(ctx, f, cycles, bs)
        self.cfg = R.make_config(hq, hkv, d, bs)
        reserve = cycles * f + 16
        # one paged cache per layer (K, V, descriptors); the page table is shared
        self.k, self.v, self.desc, self.k_scale = [], [], [], []
        for layer in range(nl):
            p = inputs.make_decode_problem(seed + 1000 * layer, B, hq, hkv, d, bs, ctx,
                                           reserve_tokens=reserve, paged=wl["paged"],
                                           device=device, topk=[1] * B)
            self.k.append(p.k_cache)
            self.v.append(p.v_cache)
            self.desc.append(torch.zeros(p.num_pages, hkv, 2, d, dtype=torch.bfloat16,
                                         device=device))
            self.k_scale.append(p.k_scale)
            self.page_table = p.page_table
            del p
        self.max_pages = int(self.page_table.shape[1])
        self.num_pages = int(self.k[0].shape[0])
        self.max_topk = self.sched.max_topk()
        self.ws = torch.empty(R.resa_workspace_size(self.cfg, B, self.max_pages, f),
                              dtype=torch.uint8, device=device)
        R.resa_workspace_init(self.ws)
        # per-step sequence lengths / top-k rows (16-byte aligned rows)
        nsteps = cycles * f
        Bp = self.sched.Bpad
        sl = torch.zeros(nsteps + 1, Bp, dtype=torch.int32)
        tk = torch.zeros(nsteps + 1, Bp, dtype=torch.int32)
        sl[nsteps, :B] = torch.tensor(ctx)
        for c in range(cycles):
            for s in range(f - 1):
                Ls = self.sched.decode_L(c, s)
                sl[c * f + s, :B] = torch.tensor(Ls)
                tk[c * f + s, :B] = torch.tensor([topk_rule(x, bs) for x in Ls])
            sl[c * f + f - 1, :B] = torch.tensor(self.sched.rect_L(c))
        self.seq_len = sl.to(device)
        self.topk = tk.to(device)
        # build the block key cache of the prefilled context (row nsteps = ctx)
        for layer in range(nl):
            R.resa_build_descriptors(self.cfg, self.cache(layer, nsteps), None, self.ws)
        # inputs of every cycle, resident in HBM
        g = torch.Generator(device=device)
        g.manual_seed(seed + 77)
        self.q = torch.randn(cycles, f - 1, nl, B, hq, d, generator=g, device=device).to(torch.bfloat16)
        kk = torch.randn(cycles, f - 1, nl, B, hkv, d, generator=g, device=device)
        for layer in range(nl):
            kk[:, :, layer] *= self.k_scale[layer][None, None, None]
        self.kn = kk.to(torch.bfloat16)
        del kk
        self.vn = torch.randn(cycles, f - 1, nl, B, hkv, d, generator=g, device=device).to(torch.bfloat16)
        self.qc = torch.randn(cycles, nl, B, f, hq, d, generator=g, device=device).to(torch.bfloat16)
        self.kc = torch.randn(cycles, nl, B, f, hkv, d, generator=g, device=device).to(torch.bfloat16)
        self.vc = torch.randn(cycles, nl, B, f, hkv, d, generator=g, device=device).to(torch.bfloat16)
        # outputs: one slot per (decode step of the cycle, layer), so that every
        # step's result survives the cycle and can be read back; two sets, used
        # by alternate cycles, so that one cycle's read-back overlaps the next
        self.out = torch.empty(2, f - 1, nl, B, hq, d, device=device)
        self.rout = torch.empty(2, nl, B, f, hq, d, device=device)
        # separate allocations keep every layer's selection buffers 16-byte aligned
        self.idx = [torch.empty(B, hkv, self.max_topk + 1, dtype=torch.int32, device=device)
                    for _ in range(nl)]
        self.cnt = [torch.empty(B, hkv, dtype=torch.int32, device=device) for _ in range(nl)]
        torch.cuda.synchronize(device)

    def cache(self, layer, step_row):
        ptr = self.seq_len.data_ptr() + 4 * self.sched.Bpad * step_row
        return self.R.make_cache(self.k[layer], self.v[layer], self.desc[layer], self.page_table,
                                 ptr)

    def topk_ptr(self, step_row):
        return self.topk.data_ptr() + 4 * self.sched.Bpad * step_row

    def launch_cycle(self, c):
        """Enqueue one ReSA cycle (all layers) on the current stream."""
        R, f = self.R, self.f
        for s in range(f - 1):
            row = c * f + s
            for layer in range(self.layers):
                R.resa_decode_step(self.cfg, self.cache(layer, row), self.q[c, s, layer],
                                   self.kn[c, s, layer], self.vn[c, s, layer], self.topk_ptr(row),
                                   self.max_topk, self.out[c % 2, s, layer], None, self.idx[layer],
                                   self.cnt[layer], self.ws)
        row = c * f + f - 1
        for layer in range(self.layers):
            R.resa_rectify_attention(self.cfg, self.cache(layer, row), f, self.qc[c, layer],
                                     self.kc[c, layer], self.vc[c, layer], self.rout[c % 2, layer], None,
                                     self.ws)

    def launches_per_cycle(self):
        R = self.R
        step = R.resa_decode_step_launches(self.cfg, self.B, self.max_pages, self.num_pages)
        return self.layers * ((self.f - 1) * step +
                              R.resa_kernels_per_call("resa_rectify_attention"))

    # algorithmic bytes / flops ---------------------------------------------
    def decode_kernel_bytes(self, Ls):
        """q + K/V of the selected blocks and the current block + fp32 output."""
        B, hq, hkv, d = self.B, self.hq, self.hkv, self.d
        bs = self.bs
        kv = sum(hkv * (min(topk_rule(L, bs), (L - 1) // bs) + 1) * bs * d * 2 * 2 for L in Ls)
        return B * hq * d * 2 + kv + B * hq * d * 4

    def step_bytes(self, Ls):
        """One sparse decode step of one layer: q + descriptors of the complete
        blocks + selected K/V + output (the per-unit figure of the design notes)."""
        hkv, d = self.hkv, self.d
        desc = sum(((L - 1) // self.bs) * hkv * 2 * d * 2 for L in Ls)
        return self.decode_kernel_bytes(Ls) + desc

    def rectify_bytes_flops(self, Ls):
        hkv, hq, d, f = self.hkv, self.hq, self.d, self.f
        byts = sum(L * hkv * d * 2 * 2 for L in Ls) + len(Ls) * f * (hq * d * 2 + hq * d * 4)
        flops = sum(sum(4 * hq * d * (L - f + r + 1) for r in range(f)) for L in Ls)
        return byts, flops


# ---------------------------------------------------------------------------
# Clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = max((num(r[2]) for r in rows if num(r[2]) is not None), default=None)
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        loaded = [s for s, p in zip(sm, power) if p is not None and p > 250] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(power) if power else None}


def kernel_dram_traffic(record="decode_step_dram_traffic.json"):
    """DRAM bytes per launch of a kernel from its committed ncu record, or None
    when the kernel's sources changed since the counters were taken."""
    import hashlib
    here = os.path.dirname(os.path.abspath(__file__))
    path = os.path.join(here, "profiles", record)
    try:
        with open(path) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(here, src), "rb") as f:
                h.update(f.read())
    except (OSError, KeyError, ValueError):
        return None, None
    if h.hexdigest() != rec["sources_sha256"]:
        return None, f"kernel changed since profiles/{record}"
    return int(rec["dram_bytes_per_launch"]), f"profiles/{record} (ncu, {rec.get('workload_short', 'layer256k')})"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained",
                                                                          d["bf16_tflops"])), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


# ---------------------------------------------------------------------------
# CPU oracle sample (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------

class OracleSample:
    """One layer of the workload held by the CPU oracle.  A sample = one sparse
    decode step + one rectification row (of f), extrapolated to a full cycle of
    every layer: layers * ((f-1) * t_decode + f * t_row)."""

    def __init__(self, wl, seed, layer_state=None):
        from block_sparse_long_resa_b200 import inputs
        from oracle import oracle as O
        self.O, self.wl = O, wl
        ctx = workload_lengths(wl, seed)
        self.ctx = ctx
        B, hq, hkv, d = wl["batch"], wl["hq"], wl["hkv"], wl["d"]
        if layer_state is None:
            p = inputs.make_decode_problem(seed, B, hq, hkv, d, 16, ctx,
                                           reserve_tokens=4 * wl["f"] + 16, paged=wl["paged"],
                                           topk=[1] * B)
            self.cache = O.OracleCache(p.k_cache, p.v_cache, p.page_table, hq, hkv, d, 16)
            self.cache.build_descriptors(p.ctx_len)
            self.L0 = list(ctx)
        else:
            k, v, desc, pt, L0 = layer_state
            self.cache = O.OracleCache(k, v, pt, hq, hkv, d, 16, desc=desc)
            self.L0 = list(L0)
        self.step = 0

    def run(self):
        import numpy as np
        from block_sparse_long_resa_b200 import inputs
        wl, f, B = self.wl, self.wl["f"], self.wl["batch"]
        hq, hkv, d = wl["hq"], wl["hkv"], wl["d"]
        self.step += 1
        L = np.array([x + self.step for x in self.L0], dtype=np.int32)
        q, kn, vn = inputs.make_step_tokens(99, self.step, B, hq, hkv, d)
        topk = [topk_rule(int(x)) for x in L]
        t0 = time.perf_counter()
        self.cache.decode_step(q, kn, vn, topk, L, max(topk))
        t_dec = time.perf_counter() - t0
        qc, kc, vc = inputs.make_rectify_chunk(99 + self.step, B, f, hq, hkv, d)
        t0 = time.perf_counter()
        self.cache.rectify_rows(qc, kc, vc, L, f, [f - 1])
        t_row = time.perf_counter() - t0
        cycle_s = wl["layers"] * ((f - 1) * t_dec + f * t_row)
        return cycle_s, t_dec, t_row

    def describe(self):
        wl = self.wl
        return (f"1 of {wl['layers']} layers: one sparse decode step (append, pooling, scores, "
                f"top-k, attention) + one of {wl['f']} rectification rows, extrapolated to a "
                f"{wl['layers']}-layer cycle of {wl['f'] - 1} decode steps + 1 rectification")


def cpu_baseline(wl, seed, layer_state, samples=2):
    """The oracle on the host cores (all threads, then one thread) on a bounded
    sample of the workload; the median sample is extrapolated to a cycle."""
    from oracle import oracle as O
    s = OracleSample(wl, seed, layer_state)
    cores = O.num_threads()
    cyc = [s.run()[0] for _ in range(samples)]
    t = statistics.median(cyc)
    O.set_num_threads(1)
    try:
        t1 = s.run()[0]
    finally:
        O.set_num_threads(cores)
    tok = wl["f"] * wl["batch"]
    return {"value": tok / t, "unit": "tokens/s", "cores": cores, "samples": samples,
            "kind": "oracle", "sample": s.describe(), "s_per_cycle_extrapolated": t,
            "threads_1": {"value": tok / t1, "unit": "tokens/s", "cores": 1, "samples": 1,
                          "s_per_cycle_extrapolated": t1}}


# ---------------------------------------------------------------------------
# Arms
# ---------------------------------------------------------------------------

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from oracle import oracle as O
    wl = WORKLOADS[args.workload]
    s = OracleSample(wl, args.seed)
    for _ in range(args.warmup):
        s.run()
    runs = [s.run() for _ in range(args.steps)]
    total = sum(r[0] for r in runs)
    measured = sum(r[1] + r[2] for r in runs)
    value = args.steps * wl["f"] * wl["batch"] / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "ms_per_step_extrapolated": True,
        "sample_ms_per_step": 1e3 * measured / args.steps,
        "vs_baseline": None, "dtype": "bf16 K/V, fp32 scores, fp64 attention (CPU oracle)",
        "data": "synthetic (seeded N(0,1) q/K/V, LogNormal K channel scale, needle blocks)",
        "config": bench_config(args.workload, wl),
        "sample_note": "each step times one decode step and one rectification row of one "
                       "layer (sample_ms_per_step) and extrapolates them to the full cycle "
                       f"(ms_per_step): {wl['layers']} layers x ({wl['f'] - 1} decode steps + "
                       f"{wl['f']} rectification rows)",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": O.num_threads(),
                         "kind": "oracle", "sample": s.describe()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_resa(args):
    import torch
    rank, world, local_rank = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the CUDA library has no CPU path)")
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist = dist_setup("nccl", world)
    wl = WORKLOADS[args.workload]
    K, W = args.steps, args.warmup
    cycles = K + W
    t_setup = time.perf_counter()
    w = GpuWorkload(wl, cycles, args.seed + rank, device)
    stream = torch.cuda.Stream(device)
    graphs = []
    with torch.cuda.stream(stream):
        # one eager cycle-0 dry run is not needed: capture directly (no host syncs inside)
        for c in range(cycles):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                w.launch_cycle(c)
            graphs.append(g)
    torch.cuda.synchronize(device)
    setup_s = time.perf_counter() - t_setup

    for c in range(W):
        graphs[c].replay()
    torch.cuda.synchronize(device)
    code = w.R.resa_check_device_status(w.ws, raise_on_error=False)
    if code:
        raise SystemExit(f"device error word 0x{code:x} after warm-up")

    clocks = ClockSampler(device.index)
    clocks.start()
    barrier(dist, device)
    torch.cuda.synchronize(device)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda.nvtx.range_push("timed")  # lets a profiler capture just these launches
        ev0.record(stream)
        for c in range(W, cycles):
            graphs[c].replay()
        ev1.record(stream)
        torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(device)
    barrier(dist, device)
    clk = clocks.stop()
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, dist, device)
    tokens = K * wl["f"] * wl["batch"] * world
    value = tokens / (ms / 1e3)

    # end to end: pinned host inputs -> device, cycle graph, outputs -> pinned host
    e2e = None
    if not args.no_e2e:
        host_in = [t[W:].cpu().pin_memory() for t in (w.q, w.kn, w.vn, w.qc, w.kc, w.vc)]
        dev_in = [w.q, w.kn, w.vn, w.qc, w.kc, w.vc]
        host_out = [torch.empty_like(w.out, device="cpu").pin_memory(),
                    torch.empty_like(w.rout, device="cpu").pin_memory()]
        h2d = sum(t[0].numel() * t.element_size() for t in host_in)
        d2h = sum(t[0].numel() * t.element_size() for t in host_out)
        # Inputs go up on one copy stream, outputs come back on another, and the
        # cycles run on the compute stream: cycle c waits for its inputs, and
        # for the read-back of cycle c - 2 (the output set it reuses).
        up = torch.cuda.Stream(device)
        down = torch.cuda.Stream(device)
        n_t = cycles - W
        ev_in = [torch.cuda.Event() for _ in range(n_t)]
        ev_run = [torch.cuda.Event() for _ in range(n_t)]
        ev_out = [torch.cuda.Event() for _ in range(n_t)]
        barrier(dist, device)
        torch.cuda.synchronize(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        up.wait_stream(stream)
        down.wait_stream(stream)
        with torch.cuda.stream(up):
            for i, c in enumerate(range(W, cycles)):
                for hsrc, ddst in zip(host_in, dev_in):
                    ddst[c].copy_(hsrc[i], non_blocking=True)
                ev_in[i].record(up)
        for i, c in enumerate(range(W, cycles)):
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])
            with torch.cuda.stream(stream):
                graphs[c].replay()
            ev_run[i].record(stream)
            down.wait_event(ev_run[i])
            with torch.cuda.stream(down):
                host_out[0][c % 2].copy_(w.out[c % 2], non_blocking=True)
                host_out[1][c % 2].copy_(w.rout[c % 2], non_blocking=True)
            ev_out[i].record(down)
        stream.wait_event(ev_out[n_t - 1])
        e1.record(stream)
        torch.cuda.synchronize(device)
        e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
        e2e = {"value": tokens / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms / K,
               "copies": "per cycle: q/k/v of every decode step and the rectification chunk "
                         "in; every decode step's output (f-1 per layer) and the rectified "
                         "rows out; copies in and out run on two copy streams, overlapped "
                         "with the neighbouring cycles' compute"}

    code = w.R.resa_check_device_status(w.ws, raise_on_error=False)

    # live per-kernel timing on the same data (last decode step's block lists)
    bd = kernel_breakdown(w, stream, device, args.breakdown_reps)

    hbm_peak, bf16_peak, bf16_sus, peak_src = measured_peaks()
    last_dec_L = w.sched.decode_L(cycles - 1, wl["f"] - 2)
    fused = w.R.resa_decode_step_launches(w.cfg, w.B, w.max_pages, w.num_pages) == 1
    if fused:
        # the fused decode step is one kernel: q + descriptors + selected K/V + output
        dec_bytes = w.step_bytes(last_dec_L)
        dec_us = bd["decode_step_us"]
        traffic, traffic_src = kernel_dram_traffic("decode_step_dram_traffic.json")
        kname = "decode_step_kernel (resa_decode_step, one launch per step)"
    else:
        dec_bytes = w.decode_kernel_bytes(last_dec_L)
        dec_us = bd["sparse_decode_us"]
        traffic, traffic_src = kernel_dram_traffic("sparse_decode_dram_traffic.json")
        kname = "sparse_decode_kernel (resa_sparse_decode)"
    dec_gbs = dec_bytes / (dec_us * 1e-6) / 1e9
    roofline = {"kernel": kname, "bound": "hbm",
                "achieved": dec_gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": dec_gbs / hbm_peak, "traffic": traffic, "traffic_source": traffic_src,
                "algorithmic_bytes_per_launch": dec_bytes,
                "launch_us": dec_us, "peak_source": peak_src,
                "isolated_launch_us": bd.get("decode_step_isolated_us") if fused else None,
                "isolated_frac": (dec_bytes / (bd["decode_step_isolated_us"] * 1e-6) / 1e9 / hbm_peak
                                  if fused else None),
                "peak_kind": "burst copy (MEASURED_PEAKS hbm_gbs)"}
    # whole-step roofline: algorithmic bytes of every kernel in the cycle
    cyc_bytes = 0
    for c in range(W, cycles):
        for s in range(wl["f"] - 1):
            cyc_bytes += wl["layers"] * w.step_bytes(w.sched.decode_L(c, s))
        rb, _ = w.rectify_bytes_flops(w.sched.rect_L(c))
        cyc_bytes += wl["layers"] * rb
    step_gbs = cyc_bytes / (ms_local / 1e3) / 1e9
    rb, rflops = w.rectify_bytes_flops(w.sched.rect_L(cycles - 1))
    rect = {"us_per_layer": bd["rectify_us"],
            "tflops": rflops / (bd["rectify_us"] * 1e-6) / 1e12,
            "hbm_gbs": rb / (bd["rectify_us"] * 1e-6) / 1e9}
    rect["frac_of_bf16_peak"] = rect["tflops"] / bf16_peak
    rect["frac_of_hbm_peak"] = rect["hbm_gbs"] / hbm_peak
    # descriptor build: every key read once, every descriptor written once
    build_bytes = sum(L * w.hkv * w.d * 2 + -(-L // w.bs) * w.hkv * 2 * w.d * 2
                      for L in last_dec_L)
    build = {"us_per_layer": bd["build_descriptors_us"],
             "hbm_gbs": build_bytes / (bd["build_descriptors_us"] * 1e-6) / 1e9}
    build["frac_of_hbm_peak"] = build["hbm_gbs"] / hbm_peak

    dense = extra = None
    if not args.no_extra:
        dense = dense_baseline(stream, device, args.seed + 500, args.breakdown_reps, hbm_peak)
        extra = {}
        for name in EXTRA_WORKLOADS:
            if name != args.workload:
                extra[name] = workload_block(name, stream, device, args.seed + 700, 3, hbm_peak)
        extra["stagger64k"] = stagger_block(stream, device, args.seed + 700, 3, hbm_peak)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        L_state = w.sched.decode_L(cycles - 1, wl["f"] - 2)
        state = (w.k[0].cpu(), w.v[0].cpu(), w.desc[0].cpu(), w.page_table.cpu(),
                 [x for x in L_state])
        cpu = cpu_baseline(wl, args.seed, state)

    per_token_us = 1e3 * (ms if world == 1 else ms_local) / K / wl["f"]  # one sequence's token latency
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 (K/V/q), fp32 accumulate and output",
        "data": "synthetic (seeded N(0,1) q/K/V, LogNormal K channel scale, needle blocks)",
        "config": bench_config(args.workload, wl),
        "execution": f"one CUDA graph per cycle; {world} replica(s)",
        "us_per_token": per_token_us,
        "roofline": roofline,
        "step_roofline": {"algorithmic_bytes_per_step": cyc_bytes / K, "achieved": step_gbs,
                          "peak": hbm_peak, "unit": "GB/s", "frac": step_gbs / hbm_peak},
        "rectify": rect,
        "build_descriptors": build,
        "kernel_breakdown_us": bd,
        "decode_step_path": "fused (1 launch)" if fused else "3 launches",
        "sparse_vs_dense_step_speedup": bd["dense_decode_us"] / bd["decode_step_us"],
        "dense_baseline": dense,
        "workloads": extra,
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": K * w.launches_per_cycle(),
        "cpu_baseline": cpu,
        "device_error_word": code,
        "setup_s": setup_s,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs
    if dist is not None:
        dist.destroy_process_group()
    return 0


def kernel_breakdown(w, stream, device, reps):
    """Average device time per call of each entry point, on the workload's own
    data, from CUDA-graph replays of one call per layer timed with events."""
    import torch
    R = w.R
    c = w.cycles - 1
    row = c * w.f + w.f - 2          # last decode step of the last cycle
    rrow = c * w.f + w.f - 1

    rounds = max(1, -(-28 // w.layers))   # >= 28 launches per graph: replay overhead amortised

    def timed(enqueue, calls):
        calls *= rounds
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for _ in range(rounds):
                    enqueue()
            g.replay()
            torch.cuda.synchronize(device)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize(device)
        return 1e3 * e0.elapsed_time(e1) / (reps * calls)

    n = w.layers
    res = {}
    res["sparse_decode_us"] = timed(lambda: [R.resa_sparse_decode(
        w.cfg, w.cache(l, row), w.q[c, w.f - 2, l], w.idx[l], w.cnt[l], w.max_topk,
        w.out[0, w.f - 2, l], None, w.ws) for l in range(n)], n)
    scratch_idx = [torch.empty_like(t) for t in w.idx]
    scratch_cnt = [torch.empty_like(t) for t in w.cnt]
    res["select_blocks_us"] = timed(lambda: [R.resa_select_blocks(
        w.cfg, w.cache(l, row), w.q[c, w.f - 2, l], w.topk_ptr(row), w.max_topk, scratch_idx[l],
        scratch_cnt[l], None, w.ws) for l in range(n)], n)
    res["append_us"] = timed(lambda: [R.resa_append_token(
        w.cfg, w.cache(l, row), w.kn[c, w.f - 2, l], w.vn[c, w.f - 2, l], w.ws)
        for l in range(n)], n)
    res["decode_step_us"] = timed(lambda: [R.resa_decode_step(
        w.cfg, w.cache(l, row), w.q[c, w.f - 2, l], w.kn[c, w.f - 2, l], w.vn[c, w.f - 2, l],
        w.topk_ptr(row), w.max_topk, w.out[0, w.f - 2, l], None, w.idx[l], w.cnt[l], w.ws)
        for l in range(n)], n)
    # the same step with a plain kernel between launches (as a projection GEMM
    # between layers would be): no overlap with the preceding launch's tail
    z = torch.zeros(1, device=device)
    t_pair = timed(lambda: [(R.resa_decode_step(
        w.cfg, w.cache(l, row), w.q[c, w.f - 2, l], w.kn[c, w.f - 2, l], w.vn[c, w.f - 2, l],
        w.topk_ptr(row), w.max_topk, w.out[0, w.f - 2, l], None, w.idx[l], w.cnt[l], w.ws),
        z.add_(1.0)) for l in range(n)], n)
    t_plain = timed(lambda: [z.add_(1.0) for _ in range(n)], n)
    res["decode_step_isolated_us"] = t_pair - t_plain
    # dense decoding of the same step (append + attention over every position, Eq. 1)
    res["dense_decode_us"] = timed(lambda: [R.resa_dense_decode(
        w.cfg, w.cache(l, row), w.q[c, w.f - 2, l], w.kn[c, w.f - 2, l], w.vn[c, w.f - 2, l],
        w.out[0, w.f - 2, l], None, w.ws) for l in range(n)], n)
    # full descriptor rebuild of every block (idempotent on the same keys)
    res["build_descriptors_us"] = timed(lambda: [R.resa_build_descriptors(
        w.cfg, w.cache(l, row), None, w.ws) for l in range(n)], n)
    res["rectify_us"] = timed(lambda: [R.resa_rectify_attention(
        w.cfg, w.cache(l, rrow), w.f, w.qc[c, l], w.kc[c, l], w.vc[c, l], w.rout[0, l], None, w.ws)
        for l in range(n)], n)
    return res


DENSE_CONTEXTS = (16384, 65536, 262144)


def dense_baseline(stream, device, seed, reps, hbm_peak):
    """One decode step of one layer (28 q / 4 kv heads, d 128, batch 1), sparse
    (top-k 10 % + current block, Eq. 2) against dense decoding over every
    position (Eq. 1), at the context lengths of the pages' speed-up figures
    (ReSA summary §5).  Each length rotates over enough independent caches
    (at least 4x the L2 size) that every call reads its K/V from HBM."""
    import torch
    from block_sparse_long_resa_b200 import inputs
    from block_sparse_long_resa_b200 import resa as R
    from block_sparse_long_resa_b200.cache import LayerCache, workspace
    hq, hkv, d = 28, 4, 128
    cfg = R.make_config(hq, hkv, d, 16)
    rows = []
    for L0 in DENSE_CONTEXTS:
        L = L0 + 1
        copies = max(2, -(-4 * 126 * 2**20 // (L0 * hkv * d * 4)))
        caches = []
        for i in range(copies):
            p = inputs.make_decode_problem(seed + 31 * i + L0, 1, hq, hkv, d, 16, [L0],
                                           reserve_tokens=16, device=device, topk=[1])
            caches.append((LayerCache.from_problem(p, device), p.q.clone(), p.k_new.clone(),
                           p.v_new.clone()))
            del p
        ws = workspace(cfg, 1, caches[0][0].max_pages, 16, device)
        for lc, *_ in caches:
            R.resa_build_descriptors(cfg, lc.struct(), None, ws)
            lc.seq_len.fill_(L)
        k = topk_rule(L)
        tk = torch.tensor([k, 0, 0, 0], dtype=torch.int32, device=device)
        out = torch.empty(1, hq, d, device=device)
        idx = torch.empty(1, hkv, k + 1, dtype=torch.int32, device=device)
        cnt = torch.empty(1, hkv, dtype=torch.int32, device=device)
        calls = 28

        def timed(one):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    for j in range(calls):
                        one(*caches[j % copies])
                g.replay()
                torch.cuda.synchronize(device)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
            torch.cuda.synchronize(device)
            return 1e3 * e0.elapsed_time(e1) / (reps * calls)

        us_s = timed(lambda lc, q, kn, vn: R.resa_decode_step(
            cfg, lc.struct(), q, kn, vn, tk, k, out, None, idx, cnt, ws))
        us_d = timed(lambda lc, q, kn, vn: R.resa_dense_decode(
            cfg, lc.struct(), q, kn, vn, out, None, ws))
        code = R.resa_check_device_status(ws, raise_on_error=False)
        M = (L - 1) // 16
        b_s = hq * d * 2 + M * hkv * 2 * d * 2 + (k + 1) * 16 * hkv * d * 4 + hq * d * 4
        b_d = hq * d * 2 + L * hkv * d * 4 + hq * d * 4
        rows.append({"context": L0, "topk": k, "sparse_step_us": us_s, "dense_step_us": us_d,
                     "dense_over_sparse": us_d / us_s,
                     "sparse_hbm_frac": b_s / (us_s * 1e-6) / 1e9 / hbm_peak,
                     "dense_hbm_frac": b_d / (us_d * 1e-6) / 1e9 / hbm_peak,
                     "cache_copies": copies, "device_error_word": code})
        del caches, ws
        torch.cuda.empty_cache()
    return {"shape": "1 layer, 28 q / 4 kv heads, d 128, batch 1, block 16", "steps": rows,
            "bytes": "sparse: q + descriptors + selected K/V + output; dense: q + all K/V "
                     "+ output; fraction of the measured HBM copy bandwidth"}


EXTRA_WORKLOADS = ("qwen32k", "cbatch", "loop64k")


def workload_block(name, stream, device, seed, reps, hbm_peak):
    """The cycle graph of a further workload, timed alone: µs per cycle, the
    decode step's µs and roofline fraction, and the amortised µs per token."""
    import torch
    wl = WORKLOADS[name]
    cycles = 2
    w = GpuWorkload(wl, cycles, seed, device)
    graphs = []
    with torch.cuda.stream(stream):
        for c in range(cycles):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                w.launch_cycle(c)
            graphs.append(g)
        graphs[0].replay()
        graphs[1].replay()
        graphs[1].replay()
        torch.cuda.synchronize(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            graphs[1].replay()
        e1.record(stream)
    torch.cuda.synchronize(device)
    cyc_us = 1e3 * e0.elapsed_time(e1) / reps
    bd = kernel_breakdown(w, stream, device, reps)
    Ls = w.sched.decode_L(cycles - 1, wl["f"] - 2)
    fused = w.R.resa_decode_step_launches(w.cfg, w.B, w.max_pages, w.num_pages) == 1
    step_b = w.step_bytes(Ls)
    gbs = step_b / (bd["decode_step_us"] * 1e-6) / 1e9
    rb, rflops = w.rectify_bytes_flops(w.sched.rect_L(cycles - 1))
    code = w.R.resa_check_device_status(w.ws, raise_on_error=False)
    per_layer_cycle = cyc_us / wl["layers"]
    res = {"description": wl["text"], "context": Ls if len(Ls) <= 4 else
           {"min": min(Ls), "max": max(Ls), "sequences": len(Ls)},
           "decode_step_us": bd["decode_step_us"], "decode_step_launches":
           1 if fused else w.R.resa_decode_step_launches(w.cfg, w.B, w.max_pages, w.num_pages),
           "decode_step_gbs": gbs, "decode_step_hbm_frac": gbs / hbm_peak,
           "dense_decode_us": bd["dense_decode_us"],
           "rectify_us": bd["rectify_us"],
           "rectify_tflops": rflops / (bd["rectify_us"] * 1e-6) / 1e12,
           "cycle_us_per_layer": per_layer_cycle,
           "amortised_us_per_token_per_layer": per_layer_cycle / wl["f"],
           "tokens_per_s": wl["batch"] * wl["f"] / (cyc_us * 1e-6),
           "kernel_breakdown_us": bd,
           "device_error_word": code}
    del graphs, w
    torch.cuda.empty_cache()
    return res


STAGGER = dict(base="loop64k", phases=[0, 8, 16, 24],
               text="the loop64k decode loop with the four sequences' cycles offset by 8 "
                    "steps: at every 8th step one sequence rectifies its last 32 tokens while "
                    "the other three decode (row-mapped calls on one cache)")


def stagger_block(stream, device, seed, reps, hbm_peak):
    """Staggered rectification inside the decode batch: per step, one
    resa_decode_step over the decoding rows and (at every 8th step) one
    resa_rectify_attention over the rectifying row, both on the same cache
    through row maps.  Reports the amortised µs per token next to the
    synchronised schedule of the same workload."""
    import torch
    wl = WORKLOADS[STAGGER["base"]]
    cycles = 2
    w = GpuWorkload(wl, cycles, seed, device)
    R = w.R
    B, f, nl, hq, hkv, d = w.B, w.f, w.layers, w.hq, w.hkv, w.d
    phase = STAGGER["phases"]
    g = torch.Generator(device=device)
    g.manual_seed(seed + 5)
    q = torch.randn(cycles, f, nl, B, hq, d, generator=g, device=device).to(torch.bfloat16)
    kn = torch.randn(cycles, f, nl, B, hkv, d, generator=g, device=device).to(torch.bfloat16)
    vn = torch.randn(cycles, f, nl, B, hkv, d, generator=g, device=device).to(torch.bfloat16)
    qc = torch.randn(cycles, f, nl, 1, f, hq, d, generator=g, device=device).to(torch.bfloat16)
    kc = torch.randn(cycles, f, nl, 1, f, hkv, d, generator=g, device=device).to(torch.bfloat16)
    vc = torch.randn(cycles, f, nl, 1, f, hkv, d, generator=g, device=device).to(torch.bfloat16)
    out = torch.empty(f, nl, B, hq, d, device=device)
    rout = torch.empty(nl, 1, f, hq, d, device=device)
    dec_rows, rect_rows, topk = [], [], []
    for t in range(cycles * f):
        rect = [b for b in range(B) if (t + phase[b]) % f == f - 1]
        dec = [b for b in range(B) if b not in rect]
        assert len(rect) <= 1
        Ls = [w.sched.ctx[b] + t + 1 for b in range(B)]
        dec_rows.append(torch.tensor(dec, dtype=torch.int32, device=device))
        rect_rows.append(torch.tensor(rect, dtype=torch.int32, device=device) if rect else None)
        tk = torch.zeros((len(dec) + 3) // 4 * 4, dtype=torch.int32)
        tk[:len(dec)] = torch.tensor([topk_rule(Ls[b]) for b in dec])
        topk.append(tk.to(device))

    def cache(layer, t, rows):
        ptr = w.seq_len.data_ptr() + 4 * w.sched.Bpad * t
        return R.make_cache(w.k[layer], w.v[layer], w.desc[layer], w.page_table, ptr, rows)

    def launch_cycle(c):
        for s in range(f):
            t = c * f + s
            n = int(dec_rows[t].numel())
            for layer in range(nl):
                R.resa_decode_step(w.cfg, cache(layer, t, dec_rows[t]), q[c, s, layer, :n],
                                   kn[c, s, layer, :n], vn[c, s, layer, :n], topk[t], w.max_topk,
                                   out[s, layer, :n], None, w.idx[layer], w.cnt[layer], w.ws)
                if rect_rows[t] is not None:
                    R.resa_rectify_attention(w.cfg, cache(layer, t, rect_rows[t]), f,
                                             qc[c, s, layer], kc[c, s, layer], vc[c, s, layer],
                                             rout[layer], None, w.ws)

    graphs = []
    with torch.cuda.stream(stream):
        for c in range(cycles):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=stream):
                launch_cycle(c)
            graphs.append(gr)
        graphs[0].replay()
        graphs[1].replay()
        graphs[1].replay()
        torch.cuda.synchronize(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            graphs[1].replay()
        e1.record(stream)
    torch.cuda.synchronize(device)
    cyc_us = 1e3 * e0.elapsed_time(e1) / reps / nl

    def timed(enqueue, calls=28):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(gr, stream=stream):
                for _ in range(calls):
                    enqueue()
            gr.replay()
            torch.cuda.synchronize(device)
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(reps):
                gr.replay()
            a1.record(stream)
        torch.cuda.synchronize(device)
        return 1e3 * a0.elapsed_time(a1) / (reps * calls)

    # the two kinds of call of the last cycle's step where sequence 0 rectifies
    t_r = 2 * f - 1
    n = int(dec_rows[t_r].numel())
    dec_us = timed(lambda: R.resa_decode_step(
        w.cfg, cache(0, t_r, dec_rows[t_r]), q[1, f - 1, 0, :n], kn[1, f - 1, 0, :n],
        vn[1, f - 1, 0, :n], topk[t_r], w.max_topk, out[f - 1, 0, :n], None, w.idx[0], w.cnt[0],
        w.ws))
    rect_us = timed(lambda: R.resa_rectify_attention(
        w.cfg, cache(0, t_r, rect_rows[t_r]), f, qc[1, f - 1, 0], kc[1, f - 1, 0],
        vc[1, f - 1, 0], rout[0], None, w.ws))
    code = R.resa_check_device_status(w.ws, raise_on_error=False)
    res = {"description": STAGGER["text"], "phases": phase, "f": f,
           "decode_step_us_3_sequences": dec_us, "rectify_us_1_sequence": rect_us,
           "cycle_us_per_layer": cyc_us,
           "amortised_us_per_token_per_layer": cyc_us / f,
           "tokens_per_s": B * f / (cyc_us * nl * 1e-6),
           "launches_per_cycle_per_layer": sum(
               R.resa_decode_step_launches(w.cfg, int(dec_rows[t].numel()), w.max_pages,
                                           w.num_pages) +
               (R.resa_kernels_per_call("resa_rectify_attention") if rect_rows[t] is not None
                else 0) for t in range(f, 2 * f)),
           "device_error_word": code}
    del graphs, w
    torch.cuda.empty_cache()
    return res


SWEEP_FRACS = (1 / 64, 1 / 32, 1 / 16, 1 / 10, 1 / 8, 1 / 4, 1 / 2, 1.0)
SWEEP_CHUNKS = (8, 16, 32, 64)


def sweep_block_size(args, bs):
    """Decode step over the selected fractions and rectification over the
    chunk lengths at one block size b; see run_sweep."""
    import torch
    from block_sparse_long_resa_b200 import resa as R
    device = torch.device("cuda", 0)
    wl = WORKLOADS[args.workload]
    w = GpuWorkload(wl, 1, args.seed, device, bs=bs)
    stream = torch.cuda.Stream(device)
    n, B = w.layers, w.B
    row = w.f - 2  # a decode step of cycle 0
    # the cycle's earlier steps first, so that the blocks they complete carry
    # their incrementally built descriptors, as in a real decode loop
    for st in range(row):
        for layer in range(n):
            R.resa_decode_step(w.cfg, w.cache(layer, st), w.q[0, st, layer], w.kn[0, st, layer],
                               w.vn[0, st, layer], w.topk_ptr(st), w.max_topk, w.out[0, st, layer],
                               None, w.idx[layer], w.cnt[layer], w.ws)
    torch.cuda.synchronize(device)
    Ls = w.sched.decode_L(0, w.f - 2)
    M = [(L - 1) // bs for L in Ls]
    rounds = max(1, -(-28 // n))

    def timed(enqueue, calls, reps=5):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for _ in range(rounds):
                    enqueue()
            g.replay()
            torch.cuda.synchronize(device)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize(device)
        return 1e3 * e0.elapsed_time(e1) / (reps * calls * rounds)

    steps = []
    for frac in SWEEP_FRACS:
        # at least 16 blocks, as the top-k rule of the workloads
        k = [min(m, max(16, int(frac * m + 0.5))) for m in M]
        kmax = max(k)
        tk = torch.zeros(w.sched.Bpad, dtype=torch.int32, device=device)
        tk[:B] = torch.tensor(k, dtype=torch.int32)
        idx = [torch.empty(B, w.hkv, kmax + 1, dtype=torch.int32, device=device) for _ in range(n)]
        cnt = [torch.empty(B, w.hkv, dtype=torch.int32, device=device) for _ in range(n)]
        us = timed(lambda: [R.resa_decode_step(
            w.cfg, w.cache(l, row), w.q[0, row, l], w.kn[0, row, l], w.vn[0, row, l], tk, kmax,
            w.out[0, row, l], None, idx[l], cnt[l], w.ws) for l in range(n)], n)
        steps.append({"s": frac, "topk": k[0] if B == 1 else k, "us_per_layer": us,
                      "launches_per_step": R.resa_decode_step_launches(w.cfg, B, w.max_pages,
                                                                       w.num_pages)})
        del idx, cnt
    t_dense = timed(lambda: [R.resa_dense_decode(
        w.cfg, w.cache(l, row), w.q[0, row, l], w.kn[0, row, l], w.vn[0, row, l],
        w.out[0, row, l], None, w.ws) for l in range(n)], n)
    fmax = max(SWEEP_CHUNKS)
    ws = torch.empty(R.resa_workspace_size(w.cfg, B, w.max_pages, fmax), dtype=torch.uint8,
                     device=device)
    R.resa_workspace_init(ws)
    g = torch.Generator(device=device)
    g.manual_seed(args.seed + 99)
    rects = []
    for f in SWEEP_CHUNKS:
        qc = torch.randn(n, B, f, w.hq, w.d, generator=g, device=device).to(torch.bfloat16)
        kc = torch.randn(n, B, f, w.hkv, w.d, generator=g, device=device).to(torch.bfloat16)
        vc = torch.randn(n, B, f, w.hkv, w.d, generator=g, device=device).to(torch.bfloat16)
        out = torch.empty(B, f, w.hq, w.d, device=device)
        us = timed(lambda: [R.resa_rectify_attention(
            w.cfg, w.cache(l, w.f - 1), f, qc[l], kc[l], vc[l], out, None, ws)
            for l in range(n)], n)
        rects.append({"f": f, "us_per_layer": us})
        del qc, kc, vc, out
    code = R.resa_check_device_status(w.ws, raise_on_error=False) | \
        R.resa_check_device_status(ws, raise_on_error=False)
    table = []
    for st in steps:
        for rc in rects:
            f = rc["f"]
            t_tok = ((f - 1) * st["us_per_layer"] + rc["us_per_layer"]) / f
            table.append({"s": st["s"], "f": f, "us_per_token_layer": t_tok,
                          "measured_vs_dense": t_tok / t_dense,
                          "eq6_bytes_vs_dense": 1 / bs + st["s"] + 1 / f})
    res = {"b": bs, "context": Ls, "dense_step_us_per_layer": t_dense, "decode_steps": steps,
           "rectification": rects, "per_token": table, "device_error_word": code}
    del w, ws
    torch.cuda.empty_cache()
    return res


def run_sweep(args):
    """Per-token cost of a ReSA cycle over (block size b, selected fraction s,
    rectification period f) on the workload's layers:
    t_token = ((f-1) t_step(s) + t_rect(f)) / f, next to the pages' memory
    model (ReSA summary §3.3, Eq. 6): bytes per token relative to dense
    decoding = 1/b (block descriptors) + s (selected K/V) + 1/f (one dense
    pass over the cache every f tokens)."""
    import torch
    torch.cuda.set_device(torch.device("cuda", 0))
    sizes = [int(x) for x in args.sweep_block_sizes.split(",")]
    out = [sweep_block_size(args, bs) for bs in sizes]
    print(json.dumps({"sweep": args.workload, "layers": WORKLOADS[args.workload]["layers"],
                      "block_sizes": out}), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    return run_resa(args)


if __name__ == "__main__":
    sys.exit(main())
