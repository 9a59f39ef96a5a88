"""Benchmark: attention TFLOP/s on one workload, as a fraction of B200 dense bf16 tensor peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the hot path over one batch of synthetic input: 3D RoPE of q and k
(osp_rope3d) followed by attention (osp_attn_full for dense workloads; for Skiparse workloads
osp_skiparse_attn, Single then Group Skip as an alternating pair).  The default workload is the
largest one-GPU configuration, the Open-Sora Plan v1.5-shaped long video: B=1, 32 heads,
head_dim 128, 16x36x64 video tokens, RoPE split 32/48/48, Skiparse k=4 Single + Group.  `value`
counts attention flops (4*B*heads*Nq*Nkv*d, summed over sets) per second of the whole step (RoPE
included), with q/k/v resident in HBM.  The same JSON line carries a per_config block: every
measured configuration (tiny, CogVideoX-2B, Open-Sora Plan dense and Skiparse, CogVideoX-5B,
long video dense and Skiparse), each timed as its own region.

Roofline denominators: the burst bf16 GEMM peak, unless the timed region lasted a second or
more under the power cap with the SM clock held below its maximum, where the sustained GEMM
peak is the like-for-like figure; the line names the one it used.

N > 1 (one process per GPU, launched by torch.distributed.run, or spawned by this script when
no launcher set WORLD_SIZE): every rank runs its own
independent copy of the workload (the (sample, head) units of attention share nothing), so
per-GPU work is fixed ("weak" scaling) and the only collectives are the timing barrier and the
max-over-ranks reduction.

--impl reference times the fp64 CPU oracle on the host cores instead (rank 0 only), on a
bounded sample of the same workload per step.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from spacetime_attention_b200 import ops, synthetic as syn  # noqa: E402

METRIC = "attention TFLOP/s and % of B200 BF16 tensor peak per config (1 GPU)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# A timed region counts as sustained (power-capped) only when it lasted at least this long AND
# the sampled SM clock sat below this fraction of its maximum with sw_power_cap active; every
# shorter or full-clock region is compared with the burst GEMM figure.
SUSTAINED_MIN_S = 1.0
SUSTAINED_CLOCK_FRAC = 0.95


def tensor_peak(peaks: dict, src: str, clocks: dict | None, region_s: float):
    """(peak TFLOP/s, description) for a tensor-bound kernel timed over `region_s` seconds with
    the sampled `clocks`: the burst bf16 GEMM figure unless the region was long and power-capped,
    where the GEMM's own sustained figure is the like-for-like denominator."""
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    sm, mx = (clocks or {}).get("sm_mhz"), (clocks or {}).get("sm_max_mhz")
    capped = ("sw_power_cap" in (clocks or {}).get("reasons", []) and sm is not None and mx
              and sm < SUSTAINED_CLOCK_FRAC * mx)
    if region_s >= SUSTAINED_MIN_S and capped:
        return sustained, (f"{src} sustained bf16 GEMM: timed region {region_s:.2f} s, power-capped at "
                           f"median {sm:.0f} of {mx:.0f} MHz")
    clk = f"median SM {sm:.0f} of {mx:.0f} MHz" if sm is not None and mx else "clocks not sampled"
    return burst, f"{src} burst bf16 GEMM: timed region {region_s:.2f} s, {clk}"


MUFU_EX2_PER_CLK_SM = 16   # ex2.approx.f32 per clock per SM (four per SM sub-partition per clock)


def exp_rate(flops: float, head_dim: int, attn_ms: float, sms: int, clocks: dict | None) -> dict:
    """The secondary bound of the attention kernel at small head_dim: one exponential per unmasked
    (query, key) score, flops / (4 d) of them, against the MUFU rate at the sampled median SM
    clock (its maximum if not sampled)."""
    mhz = (clocks or {}).get("sm_mhz") or (clocks or {}).get("sm_max_mhz") or 1965.0
    exps = flops / (4.0 * head_dim)
    achieved = exps / (attn_ms * 1e-3) / 1e12
    peak = MUFU_EX2_PER_CLK_SM * sms * float(mhz) * 1e6 / 1e12
    return {"achieved": round(achieved, 3), "peak": round(peak, 3), "unit": "Texp/s", "frac": round(achieved / peak, 4),
            "exps_per_step": exps, "peak_source": f"{MUFU_EX2_PER_CLK_SM} ex2 per clock per SM x {sms} SMs at "
                                                  f"{float(mhz):.0f} MHz"}


def tensor_or_hbm_roofline(flops: float, nbytes: float, ms: float, peaks: dict, src: str, clocks, region_s: float):
    """Roofline of a launch that may be bound by either unit: the bound is the unit whose time at
    its peak is the longer one; frac = achieved / that unit's peak."""
    pt, pt_src = tensor_peak(peaks, src, clocks, region_s)
    pb = float(peaks["hbm_gbs"])
    tflops, gbs = flops / (ms * 1e-3) / 1e12, nbytes / (ms * 1e-3) / 1e9
    t_tensor, t_hbm = flops / (pt * 1e12), nbytes / (pb * 1e9)
    if t_tensor >= t_hbm:
        roof = {"bound": "tensor", "achieved": round(tflops, 1), "peak": pt, "unit": "TFLOP/s",
                "frac": round(tflops / pt, 4), "peak_source": pt_src}
    else:
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": pb, "unit": "GB/s",
                "frac": round(gbs / pb, 4), "peak_source": f"{src} (copy bandwidth)"}
    roof["time_bound_frac"] = round(max(t_tensor, t_hbm) / (ms * 1e-3), 4)
    return roof, tflops, gbs


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("attn_fwd_kernel.cuh", "osp_device.cuh"):
        with open(os.path.join(ROOT, "spacetime_attention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kind: str = "dense"):
    """DRAM bytes per step's attention launches from the committed ncu summary of that workload
    and attention form, if it was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", f"attn_fwd_{workload}" + ("_skiparse" if kind == "skiparse" else "") + ".txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as f:
        for line in f:
            if ":" in line and not line.startswith(" "):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha") != kernel_source_sha():
        return None
    try:
        return float(kv["dram_bytes_per_step"] if "dram_bytes_per_step" in kv else kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------

def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank float over the process group (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def step_fns(w, q, k, v, qr, kr, o, launch_events=None, kind=None):
    """Returns step() running one pass of the hot path (all launches on torch's current stream):
    3D RoPE of q and k, then dense attention or the Skiparse Single + Group pair (`kind`, default
    from the workload and --attn)."""
    sp = sparse(w, kind)

    def attn():
        if sp:
            ops.skiparse_attn(qr, kr, v, w.grid, w.skiparse_k, ops.OSP_SKIP_SINGLE, o=o)
            ops.skiparse_attn(qr, kr, v, w.grid, w.skiparse_k, ops.OSP_SKIP_GROUP, o=o)
        else:
            ops.attn_full(qr, kr, v, w.grid, w.text_len, o=o)

    def step():
        ops.rope3d(q, k, w.grid, w.text_len, w.split, q_out=qr, k_out=kr)
        if launch_events is not None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            attn()
            e1.record()
            launch_events.append((e0, e1))
        else:
            attn()
    return step


ATTN_MODE = {"value": "auto"}


def sparse(w, kind=None) -> bool:
    """Skiparse pair (Single + Group) for workloads that define k, unless `kind` ("dense" /
    "skiparse") or --attn names another form."""
    if kind is not None:
        return kind == "skiparse"
    return bool(w.skiparse_k) and ATTN_MODE["value"] not in ("dense", "frame_causal", "spatial", "temporal",
                                                             "temporal_causal")


def attention_launches(w, sms: int, kind=None) -> int:
    """Kernel launches of one attention call: the attention kernel, plus the combine kernel when
    the library splits the last partial wave of (sample*set, head, 256-row block) units over KV
    ranges (the rule of osp_attn_full: units mod SMs = R > 0 and min(SMs / R, KV tiles / 2, 8) >= 2)."""
    sp = sparse(w, kind)
    k = w.skiparse_k if sp else 1
    n = (w.seq_len if not sp else w.n_video // k)
    units = -(-n // 256) * w.heads * w.B * k
    rem = units % sms
    if rem == 0:
        return 1
    ns = min(sms // rem, (-(-n // 128)) // 2, 8)
    return 2 if ns >= 2 else 1


def launches_per_step(w, sms: int = 148, kind=None) -> int:
    n = attention_launches(w, sms, kind)
    return 1 + (2 * n if sparse(w, kind) else n)


def step_flops(w, kind=None) -> float:
    return 2 * w.skiparse_flops() if sparse(w, kind) else w.dense_flops()


def run_hbm_op(args, rank, world, local_rank):
    """Time one HBM-bound row of the path alone: osp_rope3d, osp_skiparse_gather (q, k, v with
    RoPE) or osp_skiparse_scatter.  Several input sets rotate so that every launch streams its
    bytes from DRAM rather than L2.  value = algorithmic bytes / time (GB/s)."""
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = syn.WORKLOADS[args.workload]
    nset = 3
    sets = []
    for r in range(nset):
        q, k, v = (t.to(dev) for t in syn.make_qkv(w, w.seed + 101 * r))
        sets.append((q, k, v))
    esz = 2
    if args.op == "rope":
        outs = [(torch.empty_like(q), torch.empty_like(k)) for q, k, _ in sets]
        nbytes = w.rope_bytes() + (4 * w.B * w.text_len * w.heads * w.head_dim * esz)  # text rows copied
        def launch(i):
            q, k, _ = sets[i % nset]
            ops.rope3d(q, k, w.grid, w.text_len, w.split, q_out=outs[i % nset][0], k_out=outs[i % nset][1])
    else:
        if not w.skiparse_k or w.text_len:
            raise SystemExit(f"--op {args.op} needs a Skiparse workload without text tokens")
        kk = w.skiparse_k
        if args.op == "gather":
            nbytes = 3 * 2 * w.B * w.n_video * w.heads * w.head_dim * esz
            def launch(i):
                q, k, v = sets[i % nset]
                ops.skiparse_gather(q, k, v, w.grid, kk, ops.OSP_SKIP_GROUP, split=w.split)
        else:
            nbytes = 2 * w.B * w.n_video * w.heads * w.head_dim * esz
            outs = [torch.empty_like(v) for _, _, v in sets]
            def launch(i):
                _, _, v = sets[i % nset]
                ops.skiparse_scatter(v.view(w.B * kk, w.n_video // kk, w.heads, w.head_dim), w.grid, kk,
                                     ops.OSP_SKIP_GROUP, o=outs[i % nset])
    for i in range(args.warmup):
        launch(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        launch(i)
    t1.record()
    torch.cuda.synchronize()
    ops.check_status(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    peaks, src = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"metric": f"{args.op} GB/s (HBM-bound row of the path)", "value": round(world * gbs, 1), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(w.describe(), op=args.op, bytes_per_launch=nbytes,
                           l2=f"{nset} input sets rotated ({nbytes * nset / 1e6:.0f} MB)"),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                         "frac": round(gbs / float(peaks["hbm_gbs"]), 4), "traffic": None,
                         "peak_source": f"{src} (copy bandwidth)"},
            "gpu_launches": args.steps}


def cross_launches(w, text_len: int, sms: int = 148) -> int:
    """Kernel launches of one osp_attn_cross call (same split rule as attention_launches, with the
    video tokens as queries and the text tokens as keys)."""
    units = -(-w.n_video // 256) * w.heads * w.B
    rem = units % sms
    if rem == 0:
        return 1
    return 2 if min(sms // rem, (-(-text_len // 128)) // 2, 8) >= 2 else 1


def run_cross_op(args, rank, world, local_rank):
    """Time video -> text cross-attention (osp_attn_cross) alone: the workload's video tokens as
    queries, --text-len text tokens as keys and values.  Three input sets rotate (q alone is
    larger than L2 for the full-size workloads).  value = attention flops / time."""
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = syn.WORKLOADS[args.workload]
    L = args.text_len
    nset = 3
    sets = []
    for r in range(nset):
        s = w.seed + 7 + 101 * r + 17 * rank
        sets.append(tuple(syn.randn_bf16(shape, s + i).to(dev) for i, shape in enumerate(
            [(w.B, w.n_video, w.heads, w.head_dim), (w.B, L, w.heads, w.head_dim), (w.B, L, w.heads, w.head_dim)])))
    outs = [torch.empty_like(q) for q, _, _ in sets]

    def launch(i):
        q, k, v = sets[i % nset]
        ops.attn_cross(q, k, v, w.grid, o=outs[i % nset])

    for i in range(args.warmup):
        launch(i)
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        launch(i)
    t1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ops.check_status(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    peaks, src = load_peaks()
    flops = 4.0 * w.B * w.heads * w.n_video * L * w.head_dim
    nbytes = 2 * 2 * w.B * w.heads * w.head_dim * (w.n_video + L)      # q read + o written, k and v read
    roof, tflops, gbs = tensor_or_hbm_roofline(flops, nbytes, ms, peaks, src, clocks, ms * args.steps * 1e-3)
    roof.update(traffic=None, hbm_gb_s=round(gbs, 1), bytes_per_launch=nbytes)
    n_launch = cross_launches(w, L)
    return {"metric": "cross-attention TFLOP/s (video queries, text keys)", "value": round(world * tflops, 1),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict(w.describe(), op="cross", text_len=L, queries=w.n_video, flops_per_launch=flops,
                           l2=f"{nset} input sets rotated ({nset * nbytes / 1e6:.0f} MB)"),
            "roofline": roof, "clocks": clocks, "gpu_launches": n_launch * args.steps}


def run_packed_op(args, rank, world, local_rank):
    """Time a packed batch of samples of different shapes (Multi-Resolution Frame Pack):
    osp_rope3d_packed then osp_attn_packed (block-diagonal), inputs resident in HBM (larger
    than L2).  value = block-diagonal attention flops / step time."""
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = syn.PACKED_WORKLOADS[args.packed]
    q, k, v = (t.to(dev) for t in syn.make_packed_qkv(w.heads, w.head_dim, w.total, w.seed + 17 * rank))
    qr, kr, o = torch.empty_like(q), torch.empty_like(k), torch.empty_like(q)
    bounds = w.bounds
    events = []

    def step(record=False):
        ops.rope3d_packed(q, k, w.samples, w.split, q_out=qr, k_out=kr)
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
        ops.attn_packed(qr, kr, v, bounds, o=o)
        if record:
            e1.record()
            events.append((e0, e1))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step(record=True)
    t1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ops.check_status(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    attn_ms = sum(a.elapsed_time(b) for a, b in events) / len(events)
    peaks, src = load_peaks()
    flops = w.flops()
    tflops = flops / (ms * 1e-3) / 1e12
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    peak, peak_src = tensor_peak(peaks, src, clocks, ms * args.steps * 1e-3)
    nbytes = 2 * w.total * w.heads * w.head_dim
    return {"metric": "packed-batch attention TFLOP/s (Multi-Resolution Frame Pack, 1 GPU)",
            "value": round(world * tflops, 1), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(w.describe(), ops="rope3d_packed+attn_packed", flops_per_step=flops,
                           l2=f"inputs {3 * nbytes / 1e6:.0f} MB > L2 126 MiB, no flush"),
            "roofline": {"bound": "tensor", "achieved": round(attn_tflops, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(attn_tflops / peak, 4), "traffic": None,
                         "kernel": "attn_fwd_kernel (packed segment table)",
                         "peak_source": peak_src, "avg_launch_ms": round(attn_ms, 4)},
            "clocks": clocks, "gpu_launches": 2 * args.steps}


def run_variant_op(args, rank, world, local_rank):
    """Time one attention variant alone on the workload's full video grid: spatial (per-frame,
    tensor-bound), temporal (per-position over frames, HBM-bound; --causal for t' <= t) or
    frame_causal (text block + frames, tensor-bound).  Three rotating input sets."""
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = syn.WORKLOADS[args.workload]
    T, H, W = w.grid
    HW = H * W
    L = w.text_len if args.op == "frame_causal" else (args.text_len if args.op == "skiparse_text" else 0)
    N = L + w.n_video
    nset = 3
    sets = [tuple(syn.randn_bf16((w.B, N, w.heads, w.head_dim), w.seed + 11 + 101 * r + 17 * rank + i).to(dev)
                  for i in range(3)) for r in range(nset)]
    outs = [torch.empty_like(q) for q, _, _ in sets]
    if args.op == "spatial":
        launch = lambda i: ops.attn_spatial(*sets[i % nset], w.grid, o=outs[i % nset])
        pairs = w.B * T * HW * HW
    elif args.op == "temporal":
        launch = lambda i: ops.attn_temporal(*sets[i % nset], w.grid, causal=args.causal, o=outs[i % nset])
        pairs = w.B * HW * (T * (T + 1) // 2 if args.causal else T * T)
    elif args.op == "temporal_train":   # the training forward: o and the saved lse
        lses = [torch.empty((w.B * HW, w.heads, -(-T // 128) * 128), dtype=torch.float32, device=dev)
                for _ in range(nset)]
        launch = lambda i: ops.attn_temporal_train(*sets[i % nset], w.grid, causal=args.causal, o=outs[i % nset],
                                                   lse=lses[i % nset])
        pairs = w.B * HW * (T * (T + 1) // 2 if args.causal else T * T)
    elif args.op == "skiparse_text":
        kk = w.skiparse_k
        if not kk:
            raise SystemExit("--op skiparse_text needs a Skiparse workload")

        def launch(i):   # Single then Group Skip, text joined to every set
            ops.skiparse_attn(*sets[i % nset], w.grid, kk, ops.OSP_SKIP_SINGLE, o=outs[i % nset], text_len=L)
            ops.skiparse_attn(*sets[i % nset], w.grid, kk, ops.OSP_SKIP_GROUP, o=outs[i % nset], text_len=L)
        n_set = w.n_video // kk
        pairs = 2 * w.B * (w.n_video * (L + n_set) + L * N)
    else:
        launch = lambda i: ops.attn_frame_causal(*sets[i % nset], w.grid, L, o=outs[i % nset])
        pairs = w.B * (L * L + sum(HW * (L + (t + 1) * HW) for t in range(T)))
    flops = 4.0 * w.heads * w.head_dim * pairs            # unmasked (query, key) pairs only
    nbytes = 4 * w.B * N * w.heads * w.head_dim * 2       # q, k, v read once, o written once
    if args.op == "temporal_train":
        nbytes += 4 * w.B * w.n_video * w.heads           # the lse, one fp32 per token and head
    for i in range(args.warmup):
        launch(i)
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        launch(i)
    t1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ops.check_status(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    peaks, src = load_peaks()
    tflops = flops / (ms * 1e-3) / 1e12
    gbs = nbytes / (ms * 1e-3) / 1e9
    peak_t, peak_t_src = tensor_peak(peaks, src, clocks, ms * args.steps * 1e-3)
    peak_b = float(peaks["hbm_gbs"])
    if args.op in ("temporal", "temporal_train"):
        per_set = T <= 64 and (args.op == "temporal" or os.environ.get("OSP_TEMPORAL_BWD", "1") != "0")
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak_b, "unit": "GB/s",
                "frac": round(gbs / peak_b, 4), "peak_source": f"{src} (copy bandwidth)",
                "kernel": "attn_temporal_kernel" if per_set else "attn_fwd_kernel (Single Skip, k = H*W)"}
        metric = ("temporal attention training forward GB/s (o and lse)" if args.op == "temporal_train"
                  else "temporal attention GB/s (2D+1D, 1D part)")
        value, unit = gbs, "GB/s"
    else:
        roof = {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak_t, "unit": "TFLOP/s",
                "frac": round(tflops / peak_t, 4), "peak_source": peak_t_src,
                "kernel": "attn_fwd_kernel"}
        metric = {"spatial": "spatial attention TFLOP/s (2D+1D, 2D part)",
                  "frame_causal": "frame-causal attention TFLOP/s (unmasked pairs)",
                  "skiparse_text": "Skiparse + joined text TFLOP/s (Single + Group pair, unmasked pairs)"}[args.op]
        value, unit = tflops, "TFLOP/s"
    roof.update(traffic=None, bytes_per_launch=nbytes, flops_per_launch=flops)
    cfg = dict(w.describe(), op=args.op, text_len=L, l2=f"{nset} input sets rotated ({nset * nbytes / 1e6:.0f} MB)")
    if args.op in ("temporal", "temporal_train"):
        cfg["causal"] = bool(args.causal)
    return {"metric": metric, "value": round(world * value, 1), "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg, "roofline": roof,
            "clocks": clocks, "gpu_launches": args.steps * (4 if args.op == "skiparse_text" else 1),
            "tflops": round(tflops, 1), "hbm_gbs": round(gbs, 1)}


def run_backward_op(args, rank, world, local_rank):
    """Time the attention backward pass (osp_attn_backward: row sums, dK/dV kernel, dQ kernel)
    on the workload (dense, or the Skiparse Single + Group pair with --attn skiparse), after a
    training forward that saved o and lse.  value = backward flops / backward time, counting 2.5x
    the forward's flops (the five matrix products of the standard backward: S recomputed, dV, dP,
    dQ, dK)."""
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    attn = ATTN_MODE["value"]
    if attn == "packed":
        return run_packed_backward_op(args, rank, world, dev)
    w = syn.WORKLOADS[args.workload]
    if attn == "skiparse_text":
        if not sparse(w):
            raise SystemExit("--attn skiparse_text needs a Skiparse workload")
        shape = (w.B, args.text_len + w.n_video, w.heads, w.head_dim)
        q, k, v, do = (syn.randn_bf16(shape, w.seed + 17 * rank + i).to(dev) for i in range(4))
    else:
        q, k, v = (t.to(dev) for t in syn.make_qkv(w, w.seed + 17 * rank))
        do = syn.randn_bf16(tuple(q.shape), w.seed + 99 + 17 * rank).to(dev)
    causal = attn == "frame_causal"
    factor = attn in ("spatial", "temporal", "temporal_causal")
    modes = [(w.skiparse_k, ops.OSP_SKIP_SINGLE), (w.skiparse_k, ops.OSP_SKIP_GROUP)] if sparse(w) else [(1, 0)]
    L = 0 if sparse(w) else w.text_len
    text = attn == "skiparse_text"
    if text:
        L = args.text_len
    if factor:   # the factorized attention runs over the video tokens only
        q, k, v, do = (t[:, L:].contiguous() for t in (q, k, v, do))
        L = 0
        modes = [(1, 0)]
    t_causal = attn == "temporal_causal"
    if causal:
        saved = [ops.attn_frame_causal_train(q, k, v, w.grid, L)]
    elif attn == "spatial":
        saved = [ops.attn_spatial_train(q, k, v, w.grid)]
    elif factor:
        saved = [ops.attn_temporal_train(q, k, v, w.grid, causal=t_causal)]
    else:
        saved = [ops.attn_forward_train(q, k, v, w.grid, L, sparse_k=kk, mode=m) for kk, m in modes]
    grads = [tuple(torch.empty_like(q) for _ in range(3)) for _ in modes]

    def step():
        for (kk, m), (o, lse), (dq, dk, dv) in zip(modes, saved, grads):
            if causal:
                ops.attn_frame_causal_backward(q, k, v, o, do, lse, w.grid, L, dq=dq, dk=dk, dv=dv)
            elif attn == "spatial":
                ops.attn_spatial_backward(q, k, v, o, do, lse, w.grid, dq=dq, dk=dk, dv=dv)
            elif factor:
                ops.attn_temporal_backward(q, k, v, o, do, lse, w.grid, causal=t_causal, dq=dq, dk=dk, dv=dv)
            else:
                ops.attn_backward(q, k, v, o, do, lse, w.grid, L, sparse_k=kk, mode=m, dq=dq, dk=dk, dv=dv)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ops.check_status(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    peaks, src = load_peaks()
    T, H, W = w.grid
    HW = H * W
    if causal:   # unmasked (query, key) pairs only
        pairs = w.B * (L * L + sum(HW * (L + (t + 1) * HW) for t in range(T)))
    elif attn == "spatial":
        pairs = w.B * T * HW * HW
    elif factor:
        pairs = w.B * HW * (T * (T + 1) // 2 if t_causal else T * T)
    elif text:   # both modes: video queries see text + their set, text queries see everything
        n_set, N = w.n_video // w.skiparse_k, L + w.n_video
        pairs = 2 * w.B * (w.n_video * (L + n_set) + L * N)
    else:
        pairs = None
    flops = 2.5 * 4.0 * w.heads * w.head_dim * pairs if pairs is not None else 2.5 * step_flops(w)
    tflops = flops / (ms * 1e-3) / 1e12
    # algorithmic bytes: q, k, v, o, dO read and dQ, dK, dV written once (bf16), lse read (fp32)
    rows = q.shape[0] * q.shape[1] * w.heads
    nbytes = len(modes) * (8 * 2 * rows * w.head_dim + 4 * rows)
    roof, tflops, gbs = tensor_or_hbm_roofline(flops, nbytes, ms, peaks, src, clocks, ms * args.steps * 1e-3)
    per_set = attn in ("temporal", "temporal_causal") and T <= 64 and os.environ.get("OSP_TEMPORAL_BWD", "1") != "0"
    roof.update(traffic=None, bytes_per_step=nbytes,
                kernel="attn_temporal_bwd_kernel" if per_set
                else "attn_bwd_dkdv_kernel + attn_bwd_dq_kernel + attn_bwd_dvec_kernel"
                + (" (video and text query passes) + text_bwd_gather/combine" if text else ""))
    label = {"frame_causal": "frame-causal", "spatial": "spatial (per frame)", "temporal": "temporal (per position)",
             "temporal_causal": "causal temporal (per position)",
             "skiparse_text": f"skiparse pair + {L} joined text tokens (unmasked pairs)"}.get(
                 attn, "skiparse pair" if sparse(w) else "dense")
    # launches per backward call: row sums, dK/dV, dQ (or its finalize); the joined-text form runs
    # that for both query passes plus the gather and the combine
    per_call = 1 if per_set else (8 if text else 3)
    return {"metric": "attention backward TFLOP/s (2.5x forward flops)", "value": round(world * tflops, 1),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict(w.describe(), op="backward", attn=label, flops_per_step=flops,
                           l2="inputs > L2, no flush"),
            "roofline": roof, "clocks": clocks, "gpu_launches": per_call * len(modes) * args.steps}


def run_packed_backward_op(args, rank, world, dev):
    """Time the packed-batch backward (osp_attn_packed_backward: each sample's own chain rule on
    the tcgen05 kernels through the segment table) after osp_attn_packed_train.  value = 2.5x
    the block-diagonal forward flops / backward time."""
    w = syn.PACKED_WORKLOADS[args.packed]
    q, k, v = (t.to(dev) for t in syn.make_packed_qkv(w.heads, w.head_dim, w.total, w.seed + 17 * rank))
    do = syn.randn_bf16(tuple(q.shape), w.seed + 99 + 17 * rank).to(dev)
    o, lse = ops.attn_packed_train(q, k, v, w.bounds)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))

    def step():
        ops.attn_packed_backward(q, k, v, o, do, lse, w.bounds, dq=dq, dk=dk, dv=dv)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index)
    sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ops.check_status(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    peaks, src = load_peaks()
    flops = 2.5 * w.flops()
    rows = w.total * w.heads
    nbytes = 8 * 2 * rows * w.head_dim + 4 * rows
    roof, tflops, _ = tensor_or_hbm_roofline(flops, nbytes, ms, peaks, src, clocks, ms * args.steps * 1e-3)
    roof.update(traffic=None, bytes_per_step=nbytes,
                kernel="attn_bwd_dkdv_kernel + attn_bwd_dq_kernel + attn_bwd_dvec_kernel (segment table)")
    return {"metric": "packed-batch attention backward TFLOP/s (2.5x forward flops)", "value": round(world * tflops, 1),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict(w.describe(), op="backward", attn="packed", flops_per_step=flops,
                           l2="inputs > L2, no flush"),
            "roofline": roof, "clocks": clocks, "gpu_launches": 3 * args.steps}


# Every configuration of the measured workloads, each timed as its own step in the default run:
# (workload, attention form).  Tiny is launch-latency bound and reported in microseconds.
PER_CONFIG = [("tiny", "dense"), ("tiny", "skiparse"), ("cogvideox_2b", "dense"), ("open_sora_plan", "dense"),
              ("open_sora_plan", "skiparse"), ("cogvideox_5b", "dense"), ("long_video", "dense"),
              ("long_video", "skiparse")]


def _barrier(world):
    if world > 1:
        torch.distributed.barrier()


def time_steps(w, kind, q, k, v, steps: int, warmup: int, dev, world: int, local_rank: int, flush_l2: bool):
    """Times `steps` steps of the hot path on resident q, k, v (after `warmup` untimed ones):
    barrier + synchronize on both sides, CUDA events on the launching stream, clocks sampled
    during the region.  With flush_l2 every step is preceded by a write larger than L2 and timed
    by its own events (the flush is outside them).  Returns the timings and the output tensors."""
    qr, kr, o = torch.empty_like(q), torch.empty_like(k), torch.empty_like(q)
    step = step_fns(w, q, k, v, qr, kr, o, kind=kind)
    for _ in range(warmup):
        step()
    ops.check_status(dev)
    events = []
    step_timed = step_fns(w, q, k, v, qr, kr, o, launch_events=events, kind=kind)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if flush_l2 else None
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    _barrier(world)
    torch.cuda.synchronize()
    if flush_l2:
        pairs = []
        for _ in range(steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            step_timed()
            b.record()
            pairs.append((a, b))
        torch.cuda.synchronize()
        ms_total = float(sum(a.elapsed_time(b) for a, b in pairs))
    else:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(steps):
            step_timed()
        t1.record()
        torch.cuda.synchronize()
        ms_total = t0.elapsed_time(t1)
    _barrier(world)
    clocks = sampler.stop()
    ops.check_status(dev)
    ms_total = max_over_ranks(ms_total, world, dev)
    attn_ms = float(np.mean([a.elapsed_time(b) for a, b in events]))
    return {"ms_total": ms_total, "attn_ms": attn_ms, "clocks": clocks}, (qr, kr, o)


def attn_kernel_name(w, kind, sms: int) -> str:
    return "attn_fwd_kernel" + (" + attn_combine_kernel (split tail)" if attention_launches(w, sms, kind) > 1 else "")


def per_config_entry(w, kind, t: dict, steps: int, sms: int, flushed: bool) -> dict:
    """One entry of the per-config block: step time, step and attention-kernel TFLOP/s, and the
    attention kernel's fraction of the tensor peak chosen for this region's length and clocks."""
    flops = step_flops(w, kind)
    ms = t["ms_total"] / steps
    peaks, src = load_peaks()
    peak, peak_src = tensor_peak(peaks, src, t["clocks"], t["ms_total"] * 1e-3)
    attn_tf = flops / (t["attn_ms"] * 1e-3) / 1e12
    e = {"workload": w.name,
         "attn": f"skiparse k={w.skiparse_k} single+group" if sparse(w, kind) else "dense",
         "grid": "x".join(str(x) for x in w.grid), "B": w.B, "heads": w.heads, "head_dim": w.head_dim,
         "text_len": w.text_len, "seq_len": w.seq_len, "flops_per_step": flops, "steps": steps,
         "ms_per_step": round(ms, 4), "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
         "attn_ms": round(t["attn_ms"], 4), "attn_tflops": round(attn_tf, 2), "kernel": attn_kernel_name(w, kind, sms),
         "frac": round(attn_tf / peak, 4), "peak": peak, "peak_source": peak_src,
         "l2": "L2 flushed (256 MiB write) before every step, outside its events" if flushed
               else "inputs larger than L2, no flush",
         "clocks": t["clocks"], "gpu_launches": launches_per_step(w, sms, kind) * steps,
         "exp_rate": exp_rate(flops, w.head_dim, t["attn_ms"], sms, t["clocks"])}
    if w.seq_len < 4096:
        e["us_per_step"] = round(ms * 1e3, 2)
        e["note"] = "launch-latency bound; its roofline fraction is not meaningful"
    return e


def run_ours(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    w = syn.WORKLOADS[args.workload]
    kind = "skiparse" if sparse(w) else "dense"
    q_h, k_h, v_h = syn.make_qkv(w, w.seed + 17 * rank)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    in_bytes = 3 * q.numel() * q.element_size()
    flush = in_bytes < 2 * L2_BYTES

    # ---- device-timed region: K steps, inputs resident in HBM
    t, (qr, kr, o) = time_steps(w, kind, q, k, v, args.steps, args.warmup, dev, world, local_rank, flush)
    ms_total, attn_ms, clocks = t["ms_total"], t["attn_ms"], t["clocks"]

    # ---- end to end through the public API: pinned host inputs -> device -> hot path -> host.
    # Every step copies its q, k, v from pinned host memory and its o back; the copies run on
    # their own streams with double-buffered device tensors, so step i's kernels overlap the
    # upload of step i+1 and the download of step i-1 (what a host-fed caller would do).
    qp, kp, vp = (x.pin_memory() for x in (q_h, k_h, v_h))
    ops_h = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for _ in range(2)]
    dev_in = [(q, k, v), tuple(torch.empty_like(x) for x in (q, k, v))]
    dev_out = [o, torch.empty_like(o)]
    steps_pipe = [step_fns(w, *dev_in[r], qr, kr, dev_out[r], kind=kind) for r in range(2)]
    e2e_steps = max(4, min(40, args.steps))
    compute = torch.cuda.current_stream(dev)
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    up_done, comp_done, down_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_step(i):
        r = i & 1
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(comp_done[r])          # set r's previous step has consumed it
            for dst, src in zip(dev_in[r], (qp, kp, vp)):
                dst.copy_(src, non_blocking=True)
            up_done[r].record(h2d)
        compute.wait_event(up_done[r])
        if i >= 2:
            compute.wait_event(down_done[r])           # o[r] of step i-2 has been downloaded
        steps_pipe[r]()
        comp_done[r].record(compute)
        with torch.cuda.stream(d2h):
            d2h.wait_event(comp_done[r])
            ops_h[r].copy_(dev_out[r], non_blocking=True)
            down_done[r].record(d2h)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    _barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(compute)
    for i in range(e2e_steps):
        e2e_step(i)
    compute.wait_event(down_done[(e2e_steps - 1) & 1])
    compute.wait_event(down_done[(e2e_steps - 2) & 1])
    b.record(compute)
    torch.cuda.synchronize()
    _barrier(world)
    e2e_ms = max_over_ranks(a.elapsed_time(b) / e2e_steps, world, dev)
    ops.check_status(dev)
    del qp, kp, vp, ops_h, dev_in, dev_out, steps_pipe

    flops = step_flops(w, kind)
    ms_step = ms_total / args.steps
    value = world * flops * args.steps / (ms_total * 1e-3) / 1e12
    peaks, peaks_src = load_peaks()
    peak, peak_src = tensor_peak(peaks, peaks_src, clocks, ms_total * 1e-3)
    achieved = flops / (attn_ms * 1e-3) / 1e12
    traffic = profiled_traffic(w.name, kind)
    out_bytes = o.numel() * o.element_size()
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": dict(w.describe(), ops=("rope3d+skiparse_single+skiparse_group" if kind == "skiparse"
                                          else "rope3d+attn_full"),
                       skiparse_k=w.skiparse_k if kind == "skiparse" else None,
                       parallelism=f"replicas x{world} (independent samples)",
                       l2=(f"L2 flushed (256 MiB write) before every step, outside its events" if flush
                           else f"inputs {in_bytes / 1e6:.0f} MB > L2 126 MiB, no flush"),
                       flops_per_step=flops),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": attn_kernel_name(w, kind, sms), "peak_source": peak_src,
                     "frac_of_burst_peak": round(achieved / float(peaks["bf16_tflops"]), 4),
                     "frac_of_sustained_peak": round(achieved / float(peaks.get("bf16_tflops_sustained",
                                                                                 peaks["bf16_tflops"])), 4),
                     "avg_launch_ms": round(attn_ms, 4),
                     "flops_per_launch": flops,
                     "secondary": dict(exp_rate(flops, w.head_dim, attn_ms, sms, clocks),
                                       bound="mufu (one exponential per score)")},
        "e2e": {"value": round(world * flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes, "ms_per_step": round(e2e_ms, 4),
                "steps": e2e_steps, "copies": "pinned host <-> device on two copy streams, double-buffered, "
                                              "overlapping the previous/next step's kernels"},
        "gpu_launches": launches_per_step(w, sms, kind) * args.steps,
        "clocks": clocks,
    }
    del q, k, v, qr, kr, o
    torch.cuda.empty_cache()

    # ---- every other configuration, each its own timed region (1 GPU runs only)
    if world == 1 and not args.no_per_config:
        block = []
        for name, kd in PER_CONFIG:
            wc = syn.WORKLOADS[name]
            if name == w.name and kd == kind:
                block.append(per_config_entry(wc, kd, t, args.steps, sms, flush))
                continue
            qc, kc, vc = (x.to(dev) for x in syn.make_qkv(wc))
            fl = 3 * qc.numel() * qc.element_size() < 2 * L2_BYTES
            steps = max(args.steps, 50) if fl else args.steps
            tc, outs = time_steps(wc, kd, qc, kc, vc, steps, args.warmup, dev, world, local_rank, fl)
            block.append(per_config_entry(wc, kd, tc, steps, sms, fl))
            del qc, kc, vc, outs
            torch.cuda.empty_cache()
        line["per_config"] = block
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_seconds)
    return line


# ------------------------------------------------------------------------------------------
# the oracle on the host cores
# ------------------------------------------------------------------------------------------

def oracle_sample(w, heads, rows: int, q, k, v):
    """One bounded sample of the hot path on the CPU oracle, for the given heads: RoPE of q and k
    (all tokens of those heads), then attention for the first `rows` query tokens (dense), or the
    first rows/k slots of every set for Single and Group Skip (Skiparse).  Returns
    (attention flops done, seconds in RoPE, seconds in attention)."""
    import oracle as O
    heads = list(heads)
    t0 = time.perf_counter()
    qf = q[:, :, heads].to(torch.float64).numpy()
    kf = k[:, :, heads].to(torch.float64).numpy()
    vf = v[:, :, heads].to(torch.float64).numpy()
    qr = O.round_to_bf16(O.rope3d_ref(qf, w.grid, w.text_len, w.split, w.theta))
    kr = O.round_to_bf16(O.rope3d_ref(kf, w.grid, w.text_len, w.split, w.theta))
    t1 = time.perf_counter()
    nh = len(heads)
    if not sparse(w):
        O.attn_ref(qr, kr, vf, rows=np.arange(rows))
        fl = 4.0 * w.B * nh * rows * w.seq_len * w.head_dim
    else:
        fl = 0.0
        n_set = w.n_video // w.skiparse_k
        per = max(1, rows // w.skiparse_k)
        for mode in (O.SKIP_SINGLE, O.SKIP_GROUP):
            sets = O.skiparse_sets(w.n_video, w.skiparse_k, mode)
            sel = [t for st in sets for t in st[:per]]
            O.skiparse_attn_ref(qr, kr, vf, w.skiparse_k, mode, rows=sel)
            fl += 4.0 * w.B * nh * len(sel) * n_set * w.head_dim
    return fl, t1 - t0, time.perf_counter() - t1


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:  # noqa: BLE001
        return os.cpu_count()


def _fit_rows(w, q, k, v, nheads: int, budget_s: float, probe=None):
    """Query rows per head such that RoPE of `nheads` heads plus their attention rows take about
    `budget_s` seconds, from a 32-row probe on one head."""
    _, tr, ta = probe or oracle_sample(w, [0], 32, q, k, v)
    per_row = ta / 32
    rows = (budget_s - nheads * tr) / max(nheads * per_row, 1e-9)
    return int(max(8, min(w.seq_len, rows)))


def cpu_baseline(w, budget_s: float = 15.0):
    """The oracle on a bounded sample of the workload: as many heads as keep their RoPE within a
    third of the budget, and as many query rows of those heads as fill the rest."""
    q, k, v = syn.make_qkv(w)
    probe = oracle_sample(w, [0], 32, q, k, v)
    nh = int(max(1, min(w.heads, (budget_s / 3) / max(probe[1], 1e-9))))
    heads = range(nh)
    rows = _fit_rows(w, q, k, v, nh, budget_s, probe)
    fl, tr, ta = oracle_sample(w, heads, rows, q, k, v)
    if tr + ta < 0.5 * budget_s and rows < w.seq_len:   # the small probe overestimated the per-row cost
        rows = int(min(w.seq_len, rows * max(1.0, (budget_s - tr) / max(ta, 1e-9))))
        fl, tr, ta = oracle_sample(w, heads, rows, q, k, v)
    return {"value": round(fl / (tr + ta) / 1e12, 6), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
            "sample": f"{w.name}: RoPE of all q/k tokens of {nh} of {w.heads} heads + fp64 attention of "
                      + (f"the first {rows // w.skiparse_k} slots of every set (Single and Group Skip)"
                         if sparse(w) else f"the first {rows} query tokens")
                      + f" of those heads; {tr + ta:.1f} s ({tr:.1f} s RoPE)"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = syn.WORKLOADS[args.workload]
    q, k, v = syn.make_qkv(w)
    # one head per step (rotating), rows sized so that warm-up + timed steps end in ~2.5 minutes
    per_step_s = max(0.05, 150.0 / max(1, args.steps + args.warmup))
    rows = _fit_rows(w, q, k, v, 1, per_step_s)
    for i in range(args.warmup):
        oracle_sample(w, [i % w.heads], rows, q, k, v)
    fl = tt = 0.0
    for i in range(args.steps):
        f, tr, ta = oracle_sample(w, [i % w.heads], rows, q, k, v)
        fl += f
        tt += tr + ta
    value = fl / tt / 1e12
    sample = (f"{w.name}, per step: one head (rotating), RoPE of its q/k tokens + fp64 attention of "
              + (f"the first {rows // w.skiparse_k} slots of every set (Single and Group Skip)" if sparse(w)
                 else f"the first {rows} query tokens"))
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(w.describe(), ops="oracle: rope3d_ref + attn_ref (sampled)"),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def spawn_ranks(n: int, argv) -> int:
    """Runs this script under torch.distributed.run with n local ranks; returns its exit status."""
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_video", choices=sorted(syn.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--attn", default="auto",
                    choices=["auto", "dense", "skiparse", "frame_causal", "spatial", "temporal", "temporal_causal",
                             "skiparse_text", "packed"],
                    help="Skiparse workloads: time the Single+Group pair (auto/skiparse) or dense attention; "
                         "frame_causal / spatial / temporal / temporal_causal / skiparse_text (the pair with "
                         "--text-len text tokens joined) / packed (the --packed batch): that backward "
                         "(--op backward)")
    ap.add_argument("--op", default="step",
                    choices=["step", "rope", "gather", "scatter", "cross", "packed", "spatial", "temporal",
                             "temporal_train", "frame_causal", "skiparse_text", "backward"],
                    help="step: the whole hot path (default); rope/gather/scatter: one HBM-bound row alone; "
                         "cross: video -> text cross-attention alone; packed: a packed batch of mixed shapes")
    ap.add_argument("--packed", default="frame_pack_cog2b", choices=sorted(syn.PACKED_WORKLOADS),
                    help="--op packed: the packed batch")
    ap.add_argument("--text-len", type=int, default=226, help="--op cross / skiparse_text: text tokens")
    ap.add_argument("--causal", action="store_true", help="--op temporal / temporal_train: causal in time")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU oracle baseline budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="step: skip the per-config block")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.attn in ("frame_causal", "spatial", "temporal", "temporal_causal", "skiparse_text",
                     "packed") and args.op != "backward":
        ap.error(f"--attn {args.attn} applies to --op backward (use --op {args.attn.split('_')[0]} for the forward)")
    ATTN_MODE["value"] = args.attn

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # no launcher: start one process per GPU here (127.0.0.1 rendezvous) and pass on its status
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:]))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"WORLD_SIZE={world} but --gpus={args.gpus}: launch one process per GPU (torch.distributed.run "
                 f"--nproc-per-node {args.gpus}) or pass --gpus {world}")

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        runner = {"step": run_ours, "cross": run_cross_op, "packed": run_packed_op, "spatial": run_variant_op,
                  "temporal": run_variant_op, "temporal_train": run_variant_op, "frame_causal": run_variant_op,
                  "skiparse_text": run_variant_op, "backward": run_backward_op}.get(args.op, run_hbm_op)
        line = runner(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
