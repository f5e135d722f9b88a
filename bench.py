"""Benchmark: LLSA forward + backward tokens/s at 256 x 256 pixels (N = 65536).

One step = one pass of the whole path over one batch: pool Q, K, V ->
coarse-to-fine selection -> sparse attention forward -> index transpose ->
sparse attention backward, through the C ABI of libllsa.so, on the 256^2
workload (batch 2, 6 heads, d = 64, B = 16, L = 4, K = 8, bf16 tokens).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Every (batch, head) slice is independent, so N GPUs run N independent
copies of the workload (one process per GPU, weak scaling, no data-path
collective; the process group only carries the barrier and the max over
ranks of the device time).  Rank 0 prints one JSON line.

``--impl reference`` times the CPU oracle (the plain fp64 restatement of the
method, test infrastructure) on the host cores, on a bounded sample of the
same workload, and prints the same line with "impl": "reference".

``--workload NAME`` times another forward + backward workload instead, and
``--sweep`` prints tokens/s against N for LLSA, the single-level top-K
baseline and dense attention, one JSON line per point.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# The workload the metric is quoted on (the default), and the other forward +
# backward workloads that --workload can time instead: the 128 x 128 and
# 512 x 512 training-step sizes, and at 256 x 256 the block-size and top-K
# variants the pages ablate (B = 64 runs on the CUDA-core kernels).
WORKLOADS = {
    "px256": dict(name="px256", batch=2, heads=6, H=256, W=256, d=64, B=16, L=4, K=8, sigma=4.0),
    "px128": dict(name="px128", batch=8, heads=6, H=128, W=128, d=64, B=16, L=3, K=8, sigma=4.0),
    "px512": dict(name="px512", batch=1, heads=16, H=512, W=512, d=64, B=16, L=4, K=8, sigma=8.0),
    "px256_K16": dict(name="px256_K16", batch=2, heads=6, H=256, W=256, d=64, B=16, L=4, K=16, sigma=4.0),
    "px256_B64": dict(name="px256_B64", batch=2, heads=6, H=256, W=256, d=64, B=64, L=2, K=8, sigma=4.0),
}
WORKLOAD = WORKLOADS["px256"]
METRIC_PX256 = "LLSA fwd+bwd tokens/s at 256² pixels (N=65536); % of roofline"
METRIC = METRIC_PX256
UNIT = "tokens/s"


def select_workload(name: str):
    """Makes `name` the timed workload (module state read by every arm)."""
    global WORKLOAD, METRIC
    WORKLOAD = w = WORKLOADS[name]
    METRIC = METRIC_PX256 if name == "px256" else (
        f"LLSA fwd+bwd tokens/s at {w['H']}x{w['W']} pixels (N={w['H'] * w['W']}, B={w['B']}, K={w['K']}); "
        "% of roofline")


def config_desc(extra=None):
    w = WORKLOAD
    c = {"workload": f"{w['H']}x{w['W']} pixels, N={w['H'] * w['W']}, batch {w['batch']}, {w['heads']} heads, "
                     f"d={w['d']}, B={w['B']}, L={w['L']}, K={w['K']}, enrichment at every level, bf16 tokens, "
                     f"pool+select+attn_fwd+index_transpose+attn_bwd per step",
         "tokens_per_step_per_gpu": w["batch"] * w["H"] * w["W"],
         "inputs": f"seeded smooth fields (Gaussian sigma={w['sigma']} px, +0.1 white noise), dO ~ N(0,1)",
         "l2": f"no flush: inputs larger than L2 (Q, K, V, dO = "
               f"{4 * w['batch'] * w['heads'] * w['H'] * w['W'] * w['d'] * 2 / 1e6:.0f} MB per step vs 126 MB L2)"}
    if extra:
        c.update(extra)
    return c


# ----------------------------------------------------------------- ranks

def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = False
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
        pg = True
    return rank, local, world, pg


def barrier(pg):
    if pg:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, pg, device) -> float:
    if not pg:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (every 50 ms, timestamped) read on a thread; the
    samples that fall inside the timed region (plus 100 ms either side) are
    reported.  start() returns once the first sample has arrived."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        self.thread = None
        self.t_begin = self.t_end = None
        self.ident = str(device_index)
        try:
            import torch
            u = torch.cuda.get_device_properties(device_index).uuid
            self.ident = "GPU-" + str(u)
        except Exception:
            pass

    def _reader(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def start(self):
        import threading
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.ident, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._reader, daemon=True)
        self.thread.start()
        t = time.time()
        while not self.lines and time.time() - t < 5.0 and self.proc.poll() is None:
            time.sleep(0.01)

    def begin(self):
        import datetime
        self.t_begin = datetime.datetime.now()

    def end(self):
        import datetime
        self.t_end = datetime.datetime.now()

    def stop(self):
        import datetime
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.15)   # let the sample after the region arrive
        self.proc.terminate()
        try:
            self.proc.wait(timeout=10)
        except Exception:
            self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        rows = []
        for line in list(self.lines):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(f[2]), float(f[3]), float(f[4]), f[6:10]))
            except ValueError:
                continue
        pad = datetime.timedelta(milliseconds=100)
        inside = [r for r in rows if self.t_begin and self.t_end and self.t_begin - pad <= r[0] <= self.t_end + pad]
        used = inside
        if not inside and rows and self.t_begin:
            used = [min(rows, key=lambda r: abs((r[0] - self.t_begin).total_seconds()))]
        reasons = set()
        for r in used:
            for n, val in zip(self.NAMES, r[4]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in used) if used else None,
                "sm_max_mhz": max(r[2] for r in used) if used else None,
                "reasons": sorted(reasons), "samples": len(inside),
                "samples_note": None if inside else "timed region shorter than the 50 ms sampling period: "
                                                    "nearest sample reported",
                "power_w_max": max(r[3] for r in used) if used else None}


# ------------------------------------------------------------ roofline

def tensor_peak():
    """Dense bf16 tensor peak (TFLOP/s) for a kernel timed inside a long step."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return float(m["bf16_tflops_sustained"]), "measured (MEASURED_PEAKS.json bf16_tflops_sustained)"
    except Exception:
        return 1400.0, "fallback (sustained 1.4 PFLOP/s)"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def algorithmic_bytes(stage: str, n, kl, BH: int, N: int, d: int, L: int) -> float:
    """Compulsory HBM bytes of one call of a stage (every operand read once,
    every result written once), bf16 tokens, fp32 pyramids / LSE, int32 lists."""
    tok = BH * N * d * 2
    pyr = BH * sum(n[l] for l in range(1, L + 1)) * d * 4
    idx = BH * sum(n[l] * kl[l] for l in range(1, L + 1)) * 4
    offs = BH * sum(n[l] + 1 for l in range(1, L + 1)) * 4
    lse = BH * N * 4
    if stage == "pool":          # per tensor: read x, write its pyramid
        return tok + pyr
    if stage == "select":        # read pooled Q and K of every level, write the lists
        return 2 * pyr + idx
    if stage == "attn_fwd":      # read Q, K, V, pooled K, V, lists; write O, LSE
        return 3 * tok + 2 * pyr + idx + tok + lse
    if stage == "index_transpose":   # read lists, write offsets + query lists
        return idx + offs + idx
    if stage == "attn_bwd":      # read Q, K, V, O, dO, LSE, pooled K, V, lists, CSC; write dQ, dK, dV
        return 5 * tok + lse + 2 * pyr + idx + offs + idx + 3 * tok
    raise ValueError(stage)


def keys_per_query(kl, B: int, L: int, emask: int) -> int:
    """Keys one fine query attends: the B tokens of each of its K_1 blocks and
    the K_l pooled tokens of every enriched level."""
    return kl[1] * B + sum(kl[l] for l in range(1, L + 1) if (emask >> (l - 1)) & 1)


def algorithmic_flops(stage: str, kl, BH: int, N: int, d: int, B: int, L: int, emask: int) -> float:
    """Tensor FLOPs of one attention call counted on the real (query, key)
    pairs only: forward q.k and P v (4 d per pair); backward q.k again, dP,
    dV, dQ and dK (10 d per pair)."""
    pairs = BH * N * keys_per_query(kl, B, L, emask)
    return pairs * d * (4 if stage == "attn_fwd" else 10)


def traffic_record(kernel_stage: str):
    """DRAM bytes per launch from the committed ncu summary, if the stage's
    kernel sources are unchanged since the capture; else None."""
    path = os.path.join(ROOT, "profiles", "traffic_px256.txt")
    if WORKLOAD["name"] != "px256" or not os.path.exists(path):   # the record covers the 256 x 256 workload
        return None
    digest = sources_digest(kernel_stage)
    for line in open(path):
        f = line.split()
        if len(f) >= 3 and f[0] == kernel_stage and not line.startswith("#"):
            return float(f[1]) if f[2] == digest else None
    return None


# The sources each stage's kernels are built from (the shared headers included).
STAGE_SOURCES = {
    "reorder": ("k_reorder_pool.cu",),
    "pool": ("k_reorder_pool.cu",),
    "select": ("k_select.cu",),
    "attn_fwd": ("k_attn_fwd_tc.cu",),
    "index_transpose": ("k_transpose.cu",),
    "attn_bwd": ("k_attn_bwd.cu", "k_attn_bwd_q_tc.cu", "k_attn_bwd_kv_tc.cu"),
}
SHARED_HEADERS = ("llsa_internal.cuh", "ptx.cuh", "tcgen05.cuh")


def sources_digest(stage: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hierarchical_top_sparse_b200", "csrc")
    for name in sorted(STAGE_SOURCES.get(stage, ()) + SHARED_HEADERS):
        path = os.path.join(csrc, name)
        if os.path.exists(path):
            h.update(name.encode())
            h.update(open(path, "rb").read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------ our path

STAGES = ("pool", "select", "attn_fwd", "index_transpose", "attn_bwd")


def run_ours(args, rank, local, world, pg):
    import numpy as np
    import torch

    import synthetic
    from hierarchical_top_sparse_b200 import llsa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = WORKLOAD
    p = llsa.Problem(batch=w["batch"], heads=w["heads"], height=w["H"], width=w["W"], d=w["d"], B=w["B"],
                     L=w["L"], K=w["K"], dtype=llsa.BF16)
    seed = 1000 * rank
    q, k, v = synthetic.qkv(seed, w["batch"], w["heads"], w["H"], w["W"], w["d"], w["sigma"])
    g = synthetic.upstream_grad(seed + 1, w["batch"], w["heads"], p.N, w["d"])
    host = [torch.from_numpy(x) for x in (q, k, v, g)]
    raster = [h.to(dev).to(torch.bfloat16) for h in host]
    # a DiT reorders once per network, not per attention call: untimed
    hier = [torch.empty_like(x) for x in raster]
    for src, dst in zip(raster, hier):
        llsa.reorder(p, src, dst, True)
    qd, kd, vd, gd = hier
    del raster
    pipe = llsa.Pipeline(p, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        llsa.pool(p, qd, pipe.pyrQ)
        llsa.pool(p, kd, pipe.pyrK)
        llsa.pool(p, vd, pipe.pyrV)
        if ev is not None:
            ev[1].record(stream)
        llsa.select(p, pipe.pyrQ, pipe.pyrK, pipe.idx)
        if ev is not None:
            ev[2].record(stream)
        llsa.attn_fwd(p, qd, kd, vd, pipe.pyrK, pipe.pyrV, pipe.idx, pipe.o, pipe.lse)
        if ev is not None:
            ev[3].record(stream)
        llsa.index_transpose(p, pipe.idx, pipe.offs, pipe.qlist, pipe.tscratch)
        if ev is not None:
            ev[4].record(stream)
        llsa.attn_bwd(p, qd, kd, vd, pipe.o, gd, pipe.lse, pipe.pyrK, pipe.pyrV, pipe.idx, pipe.offs, pipe.qlist,
                      pipe.dq, pipe.dk, pipe.dv, pipe.work)
        if ev is not None:
            ev[5].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if llsa.device_error() != 0:
        raise RuntimeError("a bounded device wait gave up during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    clocks = ClockSampler(dev.index)
    barrier(pg)
    torch.cuda.synchronize()
    clocks.start()
    launches0 = llsa.kernel_launches()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks.begin()
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.end()
    launches = llsa.kernel_launches() - launches0
    barrier(pg)
    clk = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    ms_total = max_over_ranks(ms_total, pg, dev)
    ms_step = ms_total / args.steps
    tokens_step = w["batch"] * p.N
    value = world * tokens_step * args.steps / (ms_total / 1e3)

    stage_ms = {}
    for j, name in enumerate(STAGES):
        stage_ms[name] = sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps)) / args.steps

    # roofline of the dominant kernel call, and of every stage
    n, kl = llsa.level_sizes(p)
    peak, peak_kind = peaks()
    stages = {}
    tpeak, tpeak_kind = tensor_peak()
    for name in STAGES:
        calls = 3 if name == "pool" else 1
        b = algorithmic_bytes(name, n, kl, p.BH, p.N, p.d, p.L) * calls
        gbs = b / (stage_ms[name] / 1e3) / 1e9
        stages[name] = {"ms": round(stage_ms[name], 4), "algorithmic_MB": round(b / 1e6, 2),
                        "achieved_GBs": round(gbs, 1), "frac": round(gbs / peak, 4)}
        if name in ("attn_fwd", "attn_bwd"):
            fl = algorithmic_flops(name, kl, p.BH, p.N, p.d, p.B, p.L, p.enrich_mask)
            tf = fl / (stage_ms[name] / 1e3) / 1e12
            stages[name].update({"algorithmic_GFLOP": round(fl / 1e9, 2), "achieved_TFLOPs": round(tf, 1),
                                 "tensor_frac": round(tf / tpeak, 4)})
    dom = max(STAGES, key=lambda s: stage_ms[s])
    traffic = traffic_record(dom)
    roof = {"bound": "hbm", "kernel": dom, "achieved": stages[dom]["achieved_GBs"], "peak": peak,
            "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else
            "fallback 6650 GB/s", "unit": "GB/s", "frac": stages[dom]["frac"],
            "traffic": traffic,
            "algorithmic_bytes_per_launch": stages[dom]["algorithmic_MB"] * 1e6 / (3 if dom == "pool" else 1)}
    # whole-step fraction: all compulsory bytes at HBM bandwidth vs the measured step
    step_bytes = sum(algorithmic_bytes(s, n, kl, p.BH, p.N, p.d, p.L) * (3 if s == "pool" else 1) for s in STAGES)
    step_floor_ms = step_bytes / (peak * 1e9) * 1e3
    # the roofline as the metric defines it: the slower of the attention FLOPs
    # at the tensor peak and the pool + select bytes at HBM bandwidth
    attn_flops = sum(algorithmic_flops(s, kl, p.BH, p.N, p.d, p.B, p.L, p.enrich_mask) for s in ("attn_fwd", "attn_bwd"))
    ps_bytes = sum(algorithmic_bytes(s, n, kl, p.BH, p.N, p.d, p.L) * (3 if s == "pool" else 1) for s in ("pool", "select"))
    t_flops_ms = attn_flops / (tpeak * 1e12) * 1e3
    t_bytes_ms = ps_bytes / (peak * 1e9) * 1e3
    literal = {"definition": "max(attention FLOPs at the bf16 tensor peak, pool+select bytes at HBM bandwidth) / step",
               "attn_GFLOP": round(attn_flops / 1e9, 2), "tensor_peak_TFLOPs": tpeak, "tensor_peak_kind": tpeak_kind,
               "pool_select_MB": round(ps_bytes / 1e6, 1), "floor_ms": round(max(t_flops_ms, t_bytes_ms), 4),
               "frac": round(max(t_flops_ms, t_bytes_ms) / ms_step, 4)}

    # reorder, timed apart from the step (a network reorders once, not per
    # attention call): Q, K, V raster -> hierarchical, O, dQ, dK, dV back
    rbufs = [torch.empty_like(qd) for _ in range(7)]
    r_src = [qd, kd, vd, pipe.o, pipe.dq, pipe.dk, pipe.dv]

    def reorders():
        for i, (src, dst) in enumerate(zip(r_src, rbufs)):
            llsa.reorder(p, src, dst, i < 3)

    for _ in range(2):
        reorders()
    r0 = torch.cuda.Event(enable_timing=True)
    r1 = torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    for _ in range(args.steps):
        reorders()
    r1.record(stream)
    torch.cuda.synchronize()
    reorder_ms = max_over_ranks(r0.elapsed_time(r1) / args.steps, pg, dev)
    rb = 7 * 2 * p.BH * p.N * p.d * 2
    reorder = {"ms": round(reorder_ms, 4), "tensors": "Q, K, V to hierarchical order; O, dQ, dK, dV back",
               "algorithmic_MB": round(rb / 1e6, 1), "achieved_GBs": round(rb / (reorder_ms / 1e3) / 1e9, 1),
               "frac": round(rb / (reorder_ms / 1e3) / 1e9 / peak, 4),
               "total_with_reorder_ms": round(ms_step + reorder_ms, 4)}
    del rbufs

    # end to end through host buffers: every step copies its Q, K, V, dO from
    # pinned host memory, runs the path and reads O, LSE, dQ, dK, dV back into
    # pinned host memory.  Steps are pipelined two deep, as a data loader would
    # run them: the copies in, the path and the copies out go on three streams,
    # and two sets of device buffers alternate, so step i + 1's inputs cross
    # PCIe while step i computes and step i - 1's results come back.
    e2e = None
    if not args.no_e2e:
        pinned_in = [llsa_pin(torch, hier_host) for hier_host in (qd, kd, vd, gd)]
        sets = [(pipe, (qd, kd, vd, gd)), (llsa.Pipeline(p, device=dev), tuple(torch.empty_like(x) for x in (qd, kd, vd, gd)))]
        outs_of = lambda pp: (pp.o, pp.lse, pp.dq, pp.dk, pp.dv)
        pinned_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs_of(pipe)]
        h2d = sum(t.numel() * t.element_size() for t in pinned_in)
        d2h = sum(t.numel() * t.element_size() for t in pinned_out)
        e_steps = max(4, min(args.steps, 12))
        s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_done = [torch.cuda.Event() for _ in range(2)]
        cmp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]

        def run_path(pp, x, st):
            qx, kx, vx, gx = x
            llsa.pool(p, qx, pp.pyrQ, st)
            llsa.pool(p, kx, pp.pyrK, st)
            llsa.pool(p, vx, pp.pyrV, st)
            llsa.select(p, pp.pyrQ, pp.pyrK, pp.idx, st)
            llsa.attn_fwd(p, qx, kx, vx, pp.pyrK, pp.pyrV, pp.idx, pp.o, pp.lse, st)
            llsa.index_transpose(p, pp.idx, pp.offs, pp.qlist, pp.tscratch, st)
            llsa.attn_bwd(p, qx, kx, vx, pp.o, gx, pp.lse, pp.pyrK, pp.pyrV, pp.idx, pp.offs, pp.qlist,
                          pp.dq, pp.dk, pp.dv, pp.work, st)

        def e2e_step(i):
            b = i & 1
            pp, x = sets[b]
            with torch.cuda.stream(s_in):
                s_in.wait_event(cmp_done[b])            # step i - 2 has read this set's inputs
                for src, dst in zip(pinned_in, x):
                    dst.copy_(src, non_blocking=True)
                in_done[b].record(s_in)
            s_cmp.wait_event(in_done[b])
            s_cmp.wait_event(out_done[b])               # step i - 2's results have left this set
            run_path(pp, x, s_cmp)
            cmp_done[b].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[b])
                for src, dst in zip(outs_of(pp), pinned_out):
                    dst.copy_(src, non_blocking=True)
                out_done[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(pg)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(s_in)
        for i in range(e_steps):
            e2e_step(i)
        a1.record(s_out)
        torch.cuda.synchronize()
        barrier(pg)
        e_ms = max_over_ranks(a0.elapsed_time(a1), pg, dev)
        e2e = {"value": round(world * tokens_step * e_steps / (e_ms / 1e3), 1), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
               "ms_per_step": round(e_ms / e_steps, 4),
               "pipelined": "2 deep: H2D, path and D2H on separate streams, two device buffer sets"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(budget_s=args.cpu_seconds)

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": config_desc({"parallelism": f"{world} independent replicas (batch x heads slices), "
                                                      "no collective"}),
                "roofline": roof,
                "step_roofline": {"bound": "hbm", "compulsory_MB": round(step_bytes / 1e6, 1),
                                  "floor_ms": round(step_floor_ms, 4), "frac": round(step_floor_ms / ms_step, 4)},
                "literal_roofline": literal, "stages": stages, "reorder": reorder, "gpu_launches": launches,
                "clocks": clk, "e2e": e2e, "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------ N sweep
#
# The shape of the pages' speed figures on this GPU: forward tokens/s of the
# attention against N for LLSA, the single-level top-K baseline and dense
# attention (the inference kernel speed-up figure), and backward tokens/s
# against N (the sparse-KV backward figure, expected roughly flat in N).
# Dense attention is LLSA with K covering every block and no enrichment: its
# selection is then trivial and only the attention is timed.

SWEEP_SIDES = (64, 128, 256, 512)
SWEEP_TOKENS = 786432           # batch x heads x N per step at every N (6 heads; 3 at 512^2)
DENSE_MAX_BLOCKS = 4096         # the tensor-core attention paths take K_1 <= 4096


def sweep_problem(llsa, side: int, mode: str):
    heads = min(6, SWEEP_TOKENS // (side * side))
    batch = SWEEP_TOKENS // (heads * side * side)
    L = 4 if side >= 256 else 3
    if mode == "llsa":
        return llsa.Problem(batch=batch, heads=heads, height=side, width=side, d=64, B=16, L=L, K=8)
    if mode == "topk_single_level":
        return llsa.Problem(batch=batch, heads=heads, height=side, width=side, d=64, B=16, L=1, K=8)
    return llsa.Problem(batch=batch, heads=heads, height=side, width=side, d=64, B=16, L=1, K=10 ** 6,
                        enrich_mask=0)


def run_sweep(args, local):
    import torch

    import synthetic
    from hierarchical_top_sparse_b200 import llsa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    out = []
    for side in SWEEP_SIDES:
        for mode in ("llsa", "topk_single_level", "dense"):
            p = sweep_problem(llsa, side, mode)
            n1 = p.N // p.B
            rec = {"sweep": "tokens/s vs N", "tokens": "query rows (batch x heads x N)", "N": p.N, "side": side,
                   "mode": mode, "batch": p.batch,
                   "heads": p.heads, "L": p.L, "K": min(p.K, n1), "enrich_mask": p.enrich_mask}
            if mode == "dense" and n1 > DENSE_MAX_BLOCKS:
                rec["skipped"] = (f"K_1 = {n1} blocks exceeds the tensor-core paths' {DENSE_MAX_BLOCKS}; "
                                  "the index list alone would be " f"{p.batch * p.heads * n1 * n1 * 4 / 1e9:.1f} GB")
                print(json.dumps(rec), flush=True)
                out.append(rec)
                continue
            q, k, v = synthetic.qkv(side, p.batch, p.heads, side, side, p.d, 4.0 if side <= 256 else 8.0)
            g = synthetic.upstream_grad(side + 1, p.batch, p.heads, p.N, p.d)
            hier = []
            for x in (q, k, v, g):
                r = torch.from_numpy(x).to(dev).to(torch.bfloat16)
                h = torch.empty_like(r)
                llsa.reorder(p, r, h, True)
                hier.append(h)
                del r
            qd, kd, vd, gd = hier
            pipe = llsa.Pipeline(p, device=dev)

            def sel():
                llsa.pool(p, qd, pipe.pyrQ)
                llsa.pool(p, kd, pipe.pyrK)
                llsa.pool(p, vd, pipe.pyrV)
                llsa.select(p, pipe.pyrQ, pipe.pyrK, pipe.idx)

            def fwd():
                llsa.attn_fwd(p, qd, kd, vd, pipe.pyrK, pipe.pyrV, pipe.idx, pipe.o, pipe.lse)

            def bwd():
                llsa.index_transpose(p, pipe.idx, pipe.offs, pipe.qlist, pipe.tscratch)
                llsa.attn_bwd(p, qd, kd, vd, pipe.o, gd, pipe.lse, pipe.pyrK, pipe.pyrV, pipe.idx, pipe.offs,
                              pipe.qlist, pipe.dq, pipe.dk, pipe.dv, pipe.work)

            parts = (fwd, bwd) if mode == "dense" else (sel, fwd, bwd)
            if mode == "dense":
                sel()                      # the full index lists, once, untimed
            steps = args.sweep_steps if mode != "dense" or side <= 128 else max(2, args.sweep_steps // 5)
            for _ in range(2):
                for f in parts:
                    f()
            torch.cuda.synchronize()
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(parts) + 1)] for _ in range(steps)]
            for i in range(steps):
                evs[i][0].record(stream)
                for j, f in enumerate(parts):
                    f()
                    evs[i][j + 1].record(stream)
            torch.cuda.synchronize()
            if llsa.device_error() != 0:
                raise RuntimeError("a bounded device wait gave up during the sweep")
            ms = [sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps)) / steps
                  for j in range(len(parts))]
            names = ("attn_fwd", "transpose+attn_bwd") if mode == "dense" else ("pool+select", "attn_fwd",
                                                                                 "transpose+attn_bwd")
            tokens = p.batch * p.heads * p.N
            rec.update({"steps": steps, "ms": {nm: round(t, 4) for nm, t in zip(names, ms)},
                        "step_ms": round(sum(ms), 4),
                        "fwd_tokens_per_s": round(tokens / ((sum(ms) - ms[-1]) / 1e3), 1),
                        "bwd_tokens_per_s": round(tokens / (ms[-1] / 1e3), 1),
                        "fwd_bwd_tokens_per_s": round(tokens / (sum(ms) / 1e3), 1),
                        "attn_paths": llsa.attn_paths(p)})
            print(json.dumps(rec), flush=True)
            out.append(rec)
            del pipe, qd, kd, vd, gd, hier
            torch.cuda.empty_cache()
    # speed-up of LLSA over dense at every N where both ran (forward: the
    # inference figure; forward + backward: a training step's attention)
    by = {(r["side"], r["mode"]): r for r in out}
    for side in SWEEP_SIDES:
        a, d = by.get((side, "llsa")), by.get((side, "dense"))
        if a and d and "skipped" not in d:
            print(json.dumps({"sweep": "speed-up vs dense", "side": side, "N": a["N"],
                              "fwd": round(a["fwd_tokens_per_s"] / d["fwd_tokens_per_s"], 2),
                              "fwd_bwd": round(a["fwd_bwd_tokens_per_s"] / d["fwd_bwd_tokens_per_s"], 2)}),
                  flush=True)


def llsa_pin(torch, t):
    h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    h.copy_(t)
    return h


# ---------------------------------------------------------- the oracle arm

def host_cpu():
    """(logical cores, CPU model) of the host."""
    model = "unknown"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def oracle_sample_step(op, inputs, rows, slices, groups=1):
    """One bounded sample of the workload on the CPU oracle: the whole path
    (pool, select, forward, transpose, backward) of ``slices`` (batch, head)
    slices, with the attention forward and backward run for ``rows`` query
    rows of each slice.  The rows are split into ``groups`` sets run
    concurrently (each set is its own oracle call over every slice), so that
    slices x groups threads keep the host cores busy.  Returns the number of
    query tokens processed."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np

    import oracle
    qh, kh, vh, gh = inputs
    sel = slice(0, slices)
    pq, pk, pv = oracle.pool(op, qh[sel]), oracle.pool(op, kh[sel]), oracle.pool(op, vh[sel])
    idx = oracle.select(op, pq, pk)
    oracle.index_transpose(op, idx)

    def attend(r):
        oracle.attn_fwd(op, qh[sel], kh[sel], vh[sel], pk, pv, idx, rows=r)
        oracle.attn_bwd(op, qh[sel], kh[sel], vh[sel], pk, pv, idx, gh[sel], rows=r)

    parts = [r for r in np.array_split(rows, groups) if len(r)]
    if len(parts) == 1:
        attend(parts[0])
    else:
        with ThreadPoolExecutor(max_workers=len(parts)) as ex:
            list(ex.map(attend, parts))
    return slices * len(rows)


def oracle_setup():
    import numpy as np

    import oracle
    import synthetic
    w = WORKLOAD
    op = oracle.Problem(H=w["H"], W=w["W"], d=w["d"], B=w["B"], L=w["L"], K=w["K"])
    q, k, v = synthetic.qkv(0, w["batch"], w["heads"], w["H"], w["W"], w["d"], w["sigma"])
    g = synthetic.upstream_grad(1, w["batch"], w["heads"], op.N, w["d"])
    BH = w["batch"] * w["heads"]
    cores, _ = host_cpu()
    slices = min(BH, cores)
    groups = max(1, -(-cores // slices))   # at least one thread per host core
    inputs = [oracle.reorder(op, x.reshape(BH, op.N, w["d"])[:slices], True) for x in (q, k, v, g)]
    return op, inputs, slices, groups


def cpu_baseline(budget_s: float = 20.0):
    import numpy as np
    op, inputs, slices, groups = oracle_setup()
    cores, model = host_cpu()
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(op.N, size=2048 * groups, replace=False))
    t = time.perf_counter()
    tokens = oracle_sample_step(op, inputs, rows, slices, groups)
    dt = time.perf_counter() - t
    reps = 1
    while time.perf_counter() - t + dt < budget_s and reps < 8:
        tokens += oracle_sample_step(op, inputs, rows, slices, groups)
        reps += 1
    dt = time.perf_counter() - t
    w = WORKLOAD
    return {"value": round(tokens / dt, 1), "unit": UNIT, "cores": slices * groups, "nproc": cores,
            "cpu_model": model, "kind": "oracle",
            "sample": f"{reps} x (pool+select+transpose of {slices} (batch,head) slices of the {w['H']}x{w['W']} "
                      f"workload, attention fwd+bwd for {len(rows)} sampled query rows of each in {groups} "
                      f"concurrent row sets; fp64 C oracle, {slices * groups} threads); tokens = query rows "
                      f"attended"}


def run_reference(args, rank, world, pg):
    if rank != 0:
        barrier(pg)
        return
    import numpy as np
    op, inputs, slices, groups = oracle_setup()
    cores, model = host_cpu()
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(op.N, size=256 * groups, replace=False))
    for _ in range(args.warmup):
        oracle_sample_step(op, inputs, rows, slices, groups)
    t = time.perf_counter()
    tokens = 0
    for _ in range(args.steps):
        tokens += oracle_sample_step(op, inputs, rows, slices, groups)
    dt = time.perf_counter() - t
    value = tokens / dt
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_desc({"parallelism": "CPU oracle on the host cores (rank 0 only)"}),
            "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": slices * groups,
                             "nproc": cores, "cpu_model": model, "kind": "oracle",
                             "sample": f"per step: pool+select+transpose of {slices} (batch,head) slices of the "
                                       f"{WORKLOAD['H']}x{WORKLOAD['W']} workload, attention fwd+bwd for "
                                       f"{len(rows)} sampled query rows of each in {groups} concurrent row sets; "
                                       f"tokens = query rows attended"},
            "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    barrier(pg)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="px256",
                    help="the workload to time (default: the one the metric is quoted on)")
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the metric's line: tokens/s against N for LLSA, single-level top-K and "
                         "dense attention, one JSON line per point (one GPU)")
    ap.add_argument("--sweep-steps", type=int, default=10)
    args = ap.parse_args()
    select_workload(args.workload)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.sweep:
        run_sweep(args, int(os.environ.get("LOCAL_RANK", "0")))
        return
    rank, local, world, pg = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world, pg)
        else:
            run_ours(args, rank, local, world, pg)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
