"""Benchmark for libsqa (decoupled-head attention on B200).

Default workload (one line of JSON from rank 0): the head-configuration
comparison at B=1, N=32768, d_head=64, non-causal, bf16 N(0,1) Q/K/V --
MHA (16,16), GQA (16,4), MQA (16,1), SQA (8,4), sSQA (8,8), xSQA (4,4),
xSMQA (4,1). One step runs sqa_attn_fwd once per head configuration; the
metric is useful attention TFLOP/s = sum 4*B*N^2*H_q*d / device time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sqa|reference]
                    [--workload headcfg32k|small|long|layer|sweep|single|linear|bwd]

`--impl reference` times the float64 CPU oracle on a bounded sample of the
same workload (rank 0 only). Other workloads print extra measurement lines
(not the headline): `small` = B=1 N=1024 (us and GB/s), `long` = N in
{65536,131072,200000}, `layer` = the causal layer x[4,16384,2048], `sweep` =
the d=128 cost grid, `single` = one configuration (for profiler captures),
`linear` = one projection GEMM, `bwd` = the attention backward (dq, dk, dv)
at the head configurations above plus a causal d=128 case.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HEAD_CONFIGS_32K = [("MHA", 16, 16), ("GQA", 16, 4), ("MQA", 16, 1), ("SQA", 8, 4), ("sSQA", 8, 8),
                    ("xSQA", 4, 4), ("xSMQA", 4, 1)]
METRIC = "attention TFLOP/s (4*B*N^2*H_q*d, halved if causal)"
L2_FLUSH_BYTES = 256 << 20     # > 126 MB L2


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_traffic_headcfg32k.json")
KERNEL_SOURCES = ["attn_fwd.cuh", "sm100.cuh"]


def kernel_source_hash():
    """sha256 over the forward attention kernel's device sources: DRAM counters
    taken from an older build of the kernel are not reported against a newer one."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "reduced_query_head_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ingest_traffic(paths):
    """ncu --csv exports named traffic_<H_q>_<H_kv>.csv -> the committed per-launch DRAM bytes file."""
    import csv
    import re
    per = {}
    for path in paths:
        m = re.search(r"traffic_(\d+)_(\d+)\.csv$", path)
        rows = list(csv.reader(open(path)))
        hi = [i for i, r in enumerate(rows) if r and r[0] == "ID"][0]
        h = rows[hi]
        mi, vi, ui = h.index("Metric Name"), h.index("Metric Value"), h.index("Metric Unit")
        unit = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "ns": 1, "us": 1e3, "usecond": 1e3,
                "msecond": 1e6, "nsecond": 1}
        # one sqa_attn_fwd call may launch two grids (the split last wave): sum over the captured launches
        vals, launches = {}, set()
        for r in rows[hi + 1:]:
            if len(r) > vi:
                launches.add(r[0])
                vals[r[mi]] = vals.get(r[mi], 0.0) + float(r[vi].replace(",", "")) * unit.get(r[ui], 1)
        per["%s/%s" % (m.group(1), m.group(2))] = {
            "dram_read_bytes": vals["dram__bytes_read.sum"], "dram_write_bytes": vals["dram__bytes_write.sum"],
            "ncu_duration_ns": vals.get("gpu__time_duration.sum"), "launches": len(launches)}
    out = {"kernel_source_sha256": kernel_source_hash(), "per_config": per,
           "command": "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
                      "--clock-control none -k regex:attn_fwd -s <launches per call> -c <launches per call> --csv "
                      "python bench.py --workload single --N 32768 --hq <H_q> --hkv <H_kv> --d 64 --steps 1 "
                      "--warmup 1 (the launches of the timed call; per-call sums)"}
    os.makedirs(os.path.dirname(TRAFFIC_FILE), exist_ok=True)
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    return out


def load_traffic(names_hq_hkv):
    """Mean DRAM bytes per attention launch over the given configs, or None if
    the counters were taken on another build of the kernel."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, "no capture"
    with open(TRAFFIC_FILE) as f:
        t = json.load(f)
    if t.get("kernel_source_sha256") != kernel_source_hash():
        return None, "capture is from an older kernel build"
    vals = []
    for H_q, H_kv in names_hq_hkv:
        e = t["per_config"].get("%d/%d" % (H_q, H_kv))
        if e is None:
            return None, "config missing from capture"
        vals.append(e["dram_read_bytes"] + e["dram_write_bytes"])
    return sum(vals) / len(vals), "ncu dram__bytes_read.sum + dram__bytes_write.sum, mean per launch"


def headline_config(world):
    """The default workload's config object (both arms report the same one)."""
    return {"workload": "head-config comparison, B=1 N=32768 d_head=64 non-causal "
                        "(MHA 16/16, GQA 16/4, MQA 16/1, SQA 8/4, sSQA 8/8, xSQA 4/4, xSMQA 4/1)",
            "global_batch": world, "seq_len": 32768, "parallelism": "dp%d" % world,
            "l2": "flushed (256 MiB write) before every timed launch"}


def attn_flops(B, N, H_q, d, causal):
    f = 4.0 * B * N * N * H_q * d
    return f / 2 if causal else f


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"bf16_tflops": j["bf16_tflops"], "bf16_tflops_sustained": j.get("bf16_tflops_sustained"),
                "hbm_gbs": j["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


# ---------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = ["-i", str(self.dev)]
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *sel, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 7:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[0]) for r in rows if num(r[0]) is not None]
        mx = [num(r[1]) for r in rows if num(r[1]) is not None]
        pw = [num(r[2]) for r in rows if num(r[2]) is not None]
        load = [s for s, p in zip(sm, pw) if p is not None and p > 300] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(pw) if pw else None}


# ---------------------------------------------------------------------- inputs
def make_attn_inputs(B, N, H_q, H_kv, d, seed, factor, device, pinned_host=False):
    import numpy as np
    import torch
    import synth
    shapes = {"q": (B, N, H_q, d), "k": (B, N, H_kv, d), "v": (B, N, H_kv, d)}
    host, dev = {}, {}
    for name, shp in shapes.items():
        h = torch.empty(shp, dtype=torch.bfloat16, pin_memory=pinned_host)
        synth.fill_bf16_into(h.data_ptr(), h.numel(), seed, name, factor)
        host[name] = h
        dev[name] = h.to(device)
    return host, dev


# ---------------------------------------------------------------------- sqa arm
def bench_sqa(args):
    import numpy as np
    import torch
    import torch.distributed as dist
    import reduced_query_head_b200 as sqa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        print("warning: --gpus %d but WORLD_SIZE=%d" % (args.gpus, world), file=sys.stderr)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    peaks = load_peaks()
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    # The global workload is `world` independent sequences (one batch element
    # per GPU); attention over (batch, group) units needs no exchange, so each
    # rank runs its own shard (weak scaling). The seed is the global batch index.
    from reduced_query_head_b200.dist import max_over_ranks, shard_range
    b_lo, b_hi = shard_range(world, rank, world)
    cfgs = []
    for name, H_q, H_kv in HEAD_CONFIGS_32K:
        B, N, d = b_hi - b_lo, 32768, 64
        host, dev = make_attn_inputs(B, N, H_q, H_kv, d, b_lo, 1.0, device, pinned_host=True)
        out = torch.empty((B, N, H_q, d), dtype=torch.bfloat16, device=device)
        out_host = torch.empty((B, N, H_q, d), dtype=torch.bfloat16, pin_memory=True)
        cfgs.append(dict(name=name, B=B, N=N, H_q=H_q, H_kv=H_kv, d=d, host=host, dev=dev, out=out,
                         out_host=out_host, flops=attn_flops(B, N, H_q, d, False)))
    scale = 1.0 / math.sqrt(64)

    def launch(c):
        sqa.sqa_attn_fwd(c["dev"]["q"], c["dev"]["k"], c["dev"]["v"], c["out"], c["B"], c["N"], c["H_q"],
                         c["H_kv"], c["d"], 0, scale, stream)

    # warm-up
    for _ in range(args.warmup):
        for c in cfgs:
            launch(c)
    torch.cuda.synchronize()
    st = sqa.sqa_device_status(stream)
    if st != sqa.SQA_OK:
        raise RuntimeError("device status after warm-up: " + sqa.sqa_status_string(st))

    # timed region: per-launch events, L2 flushed before every launch
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in cfgs]
          for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for s in range(args.steps):
        for i, c in enumerate(cfgs):
            flush.fill_(s & 0xFF)
            ev[s][i][0].record(stream)
            launch(c)
            ev[s][i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    st = sqa.sqa_device_status(stream)
    if st != sqa.SQA_OK:
        raise RuntimeError("device status after timing: " + sqa.sqa_status_string(st))
    per_cfg_ms = [[ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(args.steps)] for i in range(len(cfgs))]
    step_ms = sum(sum(x) for x in per_cfg_ms) / args.steps
    flops_step = sum(c["flops"] for c in cfgs)

    # end to end through the same entry point, host buffers in and out
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    h2d = sum(sum(t.numel() * 2 for t in c["host"].values()) for c in cfgs)
    d2h = sum(c["out"].numel() * 2 for c in cfgs)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # Uploads, kernels and downloads run on three streams so that the copies of
    # one head configuration overlap the kernels of the others (PCIe is full
    # duplex): config i+1's q/k/v go up while config i computes, and config i's
    # output comes down while config i+1 computes. A configuration's device
    # buffers are rewritten only after its previous kernel has finished.
    order = pipeline_order([sum(t.numel() * 2 for t in c["host"].values()) for c in cfgs],
                           [c["out"].numel() * 2 for c in cfgs], [c["flops"] for c in cfgs])
    up, down = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    computed = [torch.cuda.Event() for _ in cfgs]
    for c_i in range(len(cfgs)):
        computed[c_i].record(stream)
    for s in range(args.steps):
        flush.fill_((s + 1) & 0xFF)
        e2e_ev[s][0].record(stream)
        up.wait_event(e2e_ev[s][0])
        uploaded, downloaded = {}, []
        for c_i in order:
            c = cfgs[c_i]
            up.wait_event(computed[c_i])
            with torch.cuda.stream(up):
                for name in ("q", "k", "v"):
                    c["dev"][name].copy_(c["host"][name], non_blocking=True)
            ev_up = torch.cuda.Event()
            ev_up.record(up)
            uploaded[c_i] = ev_up
        for c_i in order:
            c = cfgs[c_i]
            stream.wait_event(uploaded[c_i])
            launch(c)
            computed[c_i] = torch.cuda.Event()
            computed[c_i].record(stream)
            down.wait_event(computed[c_i])
            with torch.cuda.stream(down):
                c["out_host"].copy_(c["out"], non_blocking=True)
            ev_down = torch.cuda.Event()
            ev_down.record(down)
            downloaded.append(ev_down)
        stream.wait_event(downloaded[-1])
        e2e_ev[s][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev) / args.steps

    step_ms_max, e2e_ms_max = max_over_ranks([step_ms, e2e_ms], device=device)

    value = flops_step * world / (step_ms_max * 1e-3) / 1e12
    e2e_value = flops_step * world / (e2e_ms_max * 1e-3) / 1e12
    launch_ms = step_ms / len(cfgs)
    achieved = (flops_step / len(cfgs)) / (launch_ms * 1e-3) / 1e12
    traffic, traffic_src = load_traffic([(c["H_q"], c["H_kv"]) for c in cfgs])
    alg_bytes = sum(2 * c["B"] * c["N"] * c["d"] * (2 * c["H_q"] + 2 * c["H_kv"]) for c in cfgs) / len(cfgs)
    peak = peaks["bf16_tflops"]

    result = None
    if rank == 0:
        extras = headline_extras(args, sqa, torch, device, stream, peaks) if (world == 1 and not args.no_extras) \
            else None
        cpu = cpu_baseline(seconds=args.cpu_seconds) if (world == 1 and not args.no_cpu_baseline) else None
        per = {}
        for i, c in enumerate(cfgs):
            ms = statistics.median(per_cfg_ms[i])
            per[c["name"]] = {"H_q": c["H_q"], "H_kv": c["H_kv"], "ms_median": round(ms, 4),
                              "ms_min": round(min(per_cfg_ms[i]), 4),
                              "tflops": round(c["flops"] / (ms * 1e-3) / 1e12, 1)}
        t16 = statistics.mean([per[n]["ms_median"] for n in ("MHA", "GQA", "MQA")])
        t8 = statistics.mean([per[n]["ms_median"] for n in ("SQA", "sSQA")])
        t4 = statistics.mean([per[n]["ms_median"] for n in ("xSQA", "xSMQA")])
        result = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 Q/K/V; per-rank seed)",
            "config": headline_config(world),
            "pct_of_peak": round(100.0 * value / world / peak, 1),
            "roofline": {"bound": "tensor", "kernel": "sqa::attn_fwd_kernel<64>", "achieved": round(achieved, 1),
                         "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 3),
                         "peak_source": peaks["source"] + " bf16 dense (burst; each launch timed alone)",
                         "traffic": traffic, "traffic_source": traffic_src,
                         "algorithmic_bytes_per_launch": alg_bytes},
            "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms_max, 4)},
            # attention kernel launches in the timed steps, all ranks (a call is one or two grids)
            "gpu_launches": args.steps * world * sum(
                sqa.sqa_attn_fwd_grids(c["B"], c["N"], c["H_q"], c["H_kv"], c["d"], 0) for c in cfgs),
            "clocks": clk,
            "per_config": per,
            "speedup_vs_flop_ratio": {"t16/t8": round(t16 / t8, 3), "flop_ratio_16/8": 2.0,
                                      "t16/t4": round(t16 / t4, 3), "flop_ratio_16/4": 4.0},
            "cpu_baseline": cpu,
            "extras": extras,
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


# ---------------------------------------------------------------------- headline extras
SQA_CLAIM = ("up to 3x higher throughput than MHA on sequences of 32k-200k tokens, in computation-bound "
             "scenarios (pre-training, fine-tuning, encoder tasks); hardware, model and batch not stated "
             "(\"Sparse Query Attention (SQA)\", abstract)")


def headline_extras(args, sqa, torch, device, stream, peaks):
    """The rest of the metric next to the headline, each once, L2-flushed, on this GPU:
    attention at N=200000 for MHA / SQA / xSQA (the ms-per-layer-at-200k half of the metric),
    their speed-up over MHA beside the pages' claim, four d=128 points of the cost sweep, one
    backward, one decode step, the causal layer x[4,16384,2048] and the small N=1024 case."""
    import copy
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    evict = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def sub(workload, steps, warmup, **kw):
        a = copy.copy(args)
        a.workload, a.steps, a.warmup, a.quiet = workload, steps, warmup, True
        for key, val in kw.items():
            setattr(a, key, val)
        out = []
        _bench_extra(a, sqa, torch, device, stream, flush, evict, peaks, out)
        return out

    clocks = ClockSampler(device.index or 0)
    clocks.start()
    try:
        long_all = sub("long", 3, 1, long_N=(65536, 131072, 200000))
        long = [x for x in long_all if x["N"] == 200000]
        d128 = sub("sweep", 3, 1, sweep_points={(32768, 32, 8, 0), (32768, 32, 8, 1), (65536, 16, 4, 0),
                                                (65536, 16, 4, 1)})
        bwd = sub("bwd", 5, 2, N=32768, hq=8, hkv=4, d=64, causal=0)
        dec = sub("decode", 10, 3, B=8, N=32768, d=64, decode_cfgs=("MHA", "MQA"))
        layer = sub("layer", 5, 2)
        small = sub("small", 20, 3)
    finally:
        clk = clocks.stop()
    by_hq = {(x["H_q"], x["H_kv"]): x for x in long}
    names = {(16, 16): "MHA 16/16", (8, 4): "SQA 8/4", (4, 4): "xSQA 4/4"}
    t_mha, t_sqa, t_xsqa = (by_hq[c]["ms_median"] for c in ((16, 16), (8, 4), (4, 4)))
    return {
        "long_200k": {"workload": "B=1 N=200000 d_head=64 non-causal (config 3's longest length)",
                      "per_config": {n: {k: x[k] for k in ("ms_median", "ms_min", "tflops", "pct_of_peak")}
                                     for n, x in zip(("MHA 16/16", "SQA 8/4", "xSQA 4/4"),
                                                     (by_hq[(16, 16)], by_hq[(8, 4)], by_hq[(4, 4)]))}},
        "long_65k_131k": {
            "workload": "config 3's other lengths, B=1 d_head=64 non-causal",
            "per_config": {"N=%d %s" % (x["N"], names[(x["H_q"], x["H_kv"])]):
                           {k: x[k] for k in ("ms_median", "tflops", "pct_of_peak")}
                           for x in long_all if x["N"] != 200000}},
        "speedup_over_mha_200k": {"t_MHA/t_SQA": round(t_mha / t_sqa, 3), "flop_ratio_SQA": 2.0,
                                  "t_MHA/t_xSQA": round(t_mha / t_xsqa, 3), "flop_ratio_xSQA": 4.0,
                                  "pages_claim": SQA_CLAIM},
        "d128_sweep_points": {
            "workload": "config 5 points (cost sweep, d_head=128, inputs x0.5, seed = grid index); the full "
                        "88-point sweep is --workload sweep",
            "per_point": {"N=%d H_q=%d H_kv=%d %s" % (x["N"], x["H_q"], x["H_kv"], "causal" if x["causal"] else
                                                      "non-causal"):
                          {k: x[k] for k in ("ms_median", "tflops", "pct_of_peak")} for x in d128}},
        "backward": dict(bwd[0], note="SQA 8/4, N=32768, d=64; five N*N*d products per query head"),
        "decode": {x["config"]: {k: x[k] for k in ("us_median", "GB_per_s", "frac_of_hbm")} for x in dec},
        "layer": dict(layer[0], workload="causal layer x[4,16384,2048], H_q=16 H_kv=8 d=64"),
        "small": {x["timing"]: {k: x[k] for k in ("us_median", "GB_per_s", "tflops") if k in x} for x in small},
        "clocks": clk,
    }


# ---------------------------------------------------------------------- oracle timing
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [os.cpu_count() or 1])
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(rows_per_cfg, seed=0):
    """Oracle on `rows_per_cfg` query positions (all heads) of every head config.
    Returns (useful flops, seconds)."""
    import numpy as np
    import oracle
    import synth
    N, d = 32768, 64
    flops, secs = 0.0, 0.0
    for name, H_q, H_kv in HEAD_CONFIGS_32K:
        kb = synth.bf16_bits((1, N, H_kv, d), seed, "k")
        vb = synth.bf16_bits((1, N, H_kv, d), seed, "v")
        rows = synth.sample_rows(rows_per_cfg, N, seed ^ 0x5A17)
        q = np.empty((len(rows), H_q, d), dtype=np.uint16)
        full_q = synth.bf16_bits((1, N, H_q, d), seed, "q").reshape(N, H_q, d)
        q[:] = full_q[rows]
        t0 = time.perf_counter()
        oracle.attention_rows(oracle.widen_bf16(q), oracle.widen_bf16(kb), oracle.widen_bf16(vb), rows, N,
                              False, 1.0 / math.sqrt(d))
        secs += time.perf_counter() - t0
        flops += 4.0 * len(rows) * N * H_q * d
    return flops, secs


def pipeline_order(up_bytes, down_bytes, flops):
    """Order of the head configurations in one end-to-end step.

    The pipeline's fill is the first configuration's upload and its drain the
    last one's download, so the step starts with the smallest upload and ends
    with the smallest download of the rest. In between, configurations go in
    increasing order of upload bytes per FLOP, so the upload stream stays ahead
    of the kernels. The work is the same in any order.
    """
    n = len(up_bytes)
    if n == 0:
        return []
    first = min(range(n), key=lambda i: up_bytes[i])
    rest = [i for i in range(n) if i != first]
    if not rest:
        return [first]
    last = min(rest, key=lambda i: down_bytes[i])
    middle = sorted((i for i in rest if i != last), key=lambda i: up_bytes[i] / flops[i])
    return [first] + middle + [last]


def cpu_baseline(seconds=15.0):
    # size the sample after a warm-up call (thread pool, first-touch
    # allocation); the cost per row falls as the sample grows, so rescale until
    # one sample takes at least 60% of `seconds`
    oracle_sample(8)
    rows = 256
    f, s = oracle_sample(rows)
    for _ in range(2):
        if s >= 0.6 * seconds or rows >= 16384:
            break
        rows = int(max(rows, min(16384, rows * seconds / max(s, 1e-3))))
        f, s = oracle_sample(rows)
    return {"value": round(f / s / 1e12, 6), "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": "%d query positions (all heads) of each of the 7 head configs at N=32768, d=64, "
                      "float64 numpy/BLAS; %.1f s" % (rows, s)}


def bench_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    rows = 16
    for _ in range(args.warmup):
        oracle_sample(rows)
    f_tot, s_tot = 0.0, 0.0
    for s in range(args.steps):
        f, t = oracle_sample(rows, seed=s)
        f_tot += f
        s_tot += t
    value = f_tot / s_tot / 1e12
    cores = _blas_threads()
    sample = "%d query positions (all heads) of each of the 7 head configs per step, float64 oracle" % rows
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * s_tot / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) bf16 Q/K/V)",
        "config": headline_config(int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------- extra workloads
def _time_launches(fn, reps, flush, stream, evict=None):
    """CUDA-event time of each of `reps` calls of fn, the L2 flushed before each by a write of
    `flush`. With `evict`, a read of that second buffer (also larger than L2) follows the write,
    so the dirty lines of the flush are written back before the timed region instead of inside
    it (that write-back is a sizeable part of a kernel lasting tens of microseconds)."""
    import torch
    evs = []
    for r in range(reps):
        flush.fill_(r & 0xFF)
        if evict is not None:
            evict.sum(dtype=torch.int64)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def bench_extra(args):
    import torch
    import reduced_query_head_b200 as sqa
    device = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    evict = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)   # see _time_launches
    peaks = load_peaks()
    lines = []
    clocks = ClockSampler(0)
    clocks.start()
    try:
        _bench_extra(args, sqa, torch, device, stream, flush, evict, peaks, lines)
    finally:
        clk = clocks.stop()
    print(json.dumps({"workload": args.workload, "clocks": clk}), flush=True)
    return lines


def _emit(args, line):
    if not getattr(args, "quiet", False):
        print(json.dumps(line), flush=True)


def _bench_extra(args, sqa, torch, device, stream, flush, evict, peaks, lines):
    if args.workload in ("long", "sweep"):
        if args.workload == "long":
            grid = [(N, H_q, H_kv, 64, c, 1.0, 0) for N in getattr(args, "long_N", (65536, 131072, 200000))
                    for (_, H_q, H_kv) in (("MHA", 16, 16), ("SQA", 8, 4), ("xSQA", 4, 4)) for c in (0,)]
        else:
            grid = []
            idx = 0
            for N in (32768, 65536, 131072, 200000):
                for H_q in (32, 16, 8, 4):
                    for H_kv in (8, 4, 1):
                        if H_kv <= H_q:
                            for c in (0, 1):
                                grid.append((N, H_q, H_kv, 128, c, 0.5, idx))
                            idx += 1
            points = getattr(args, "sweep_points", None)
            if points is not None:
                grid = [g for g in grid if (g[0], g[1], g[2], g[4]) in points]
        for N, H_q, H_kv, d, causal, factor, seed in grid:
            _, dev = make_attn_inputs(1, N, H_q, H_kv, d, seed, factor, device)
            out = torch.empty((1, N, H_q, d), dtype=torch.bfloat16, device=device)

            def fn():
                sqa.sqa_attn_fwd(dev["q"], dev["k"], dev["v"], out, 1, N, H_q, H_kv, d, causal, d ** -0.5, stream)
            for _ in range(args.warmup):
                fn()
            ms = _time_launches(fn, args.steps, flush, stream)
            assert sqa.sqa_device_status(stream) == 0
            fl = attn_flops(1, N, H_q, d, causal)
            med = statistics.median(ms)
            lines.append({"workload": args.workload, "N": N, "H_q": H_q, "H_kv": H_kv, "d": d, "causal": causal,
                          "ms_median": round(med, 3), "ms_min": round(min(ms), 3),
                          "tflops": round(fl / (med * 1e-3) / 1e12, 1),
                          "pct_of_peak": round(100 * fl / (med * 1e-3) / 1e12 / peaks["bf16_tflops"], 1)})
            _emit(args, lines[-1])
            del dev, out
    elif args.workload == "small":
        # config 1: B=1, N=1024, H_q=8, H_kv=4, d=64, non-causal, scale 1/8 -- latency-bound
        B, N, H_q, H_kv, d = 1, 1024, 8, 4, 64
        _, dev = make_attn_inputs(B, N, H_q, H_kv, d, 0, 1.0, device)
        out = torch.empty((B, N, H_q, d), dtype=torch.bfloat16, device=device)

        def fn():
            sqa.sqa_attn_fwd(dev["q"], dev["k"], dev["v"], out, B, N, H_q, H_kv, d, 0, 0.125, stream)
        for _ in range(max(args.warmup, 3)):
            fn()
        cold = _time_launches(fn, args.steps, flush, stream, evict)
        warm_ev = []
        for _ in range(args.steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            warm_ev.append((a, b))
        torch.cuda.synchronize()
        warm = [a.elapsed_time(b) for a, b in warm_ev]
        assert sqa.sqa_device_status(stream) == 0
        nbytes = 2 * B * N * d * (2 * H_q + 2 * H_kv)
        fl = attn_flops(B, N, H_q, d, False)
        for name, ms in (("l2_flushed", cold), ("l2_warm", warm)):
            med = statistics.median(ms)
            lines.append({"workload": "small", "timing": name, "us_median": round(med * 1e3, 2),
                          "us_min": round(min(ms) * 1e3, 2), "GB_per_s": round(nbytes / (med * 1e-3) / 1e9, 1),
                          "tflops": round(fl / (med * 1e-3) / 1e12, 1), "bytes": nbytes})
            _emit(args, lines[-1])
        # Floors of the same timing (flush, evict, events): a 4-byte torch fill (launch and
        # event overhead alone) and this library's smallest call (one 128-row tile, one key
        # tile: the kernel's fixed set-up, first loads and teardown).
        tiny = torch.empty(1, dtype=torch.int32, device=device)
        _, dev1 = make_attn_inputs(1, 128, 1, 1, d, 0, 1.0, device)
        out1 = torch.empty((1, 128, 1, d), dtype=torch.bfloat16, device=device)

        def one_tile():
            sqa.sqa_attn_fwd(dev1["q"], dev1["k"], dev1["v"], out1, 1, 128, 1, 1, d, 0, 0.125, stream)
        for _ in range(3):
            tiny.fill_(0)
            one_tile()
        floors = (("floor_fill_4_bytes", _time_launches(lambda: tiny.fill_(0), args.steps, flush, stream, evict)),
                  ("floor_attn_one_tile", _time_launches(one_tile, args.steps, flush, stream, evict)))
        assert sqa.sqa_device_status(stream) == 0
        for name, ms in floors:
            lines.append({"workload": "small", "timing": name, "us_median": round(statistics.median(ms) * 1e3, 2),
                          "us_min": round(min(ms) * 1e3, 2)})
            _emit(args, lines[-1])
    elif args.workload == "linear":
        # one projection GEMM y[M, N_out] = x[M, K] W^T (default: the layer's QKV shape)
        import synth
        M, K, N_out = args.M, args.K, args.N_out

        def mk(shape, name, factor):
            h = torch.empty(shape, dtype=torch.bfloat16)
            synth.fill_bf16_into(h.data_ptr(), h.numel(), 0, name, factor)
            return h.to(device)
        x, w = mk((M, K), "x", 1.0), mk((N_out, K), "wq", 0.02)
        y = torch.empty((M, N_out), dtype=torch.bfloat16, device=device)

        def fn():
            sqa.sqa_linear_fwd(x, w, y, M, K, N_out, stream)
        for _ in range(args.warmup):
            fn()
        ms = _time_launches(fn, args.steps, flush, stream)
        assert sqa.sqa_device_status(stream) == 0
        med = statistics.median(ms)
        fl = 2.0 * M * K * N_out
        lines.append({"workload": "linear", "M": M, "K": K, "N_out": N_out, "ms_median": round(med, 4),
                      "tflops": round(fl / (med * 1e-3) / 1e12, 1),
                      "pct_of_peak": round(100 * fl / (med * 1e-3) / 1e12 / peaks["bf16_tflops"], 1)})
        _emit(args, lines[-1])
    elif args.workload == "single":
        # one attention configuration, e.g. for a profiler capture
        N, H_q, H_kv, d, causal = args.N, args.hq, args.hkv, args.d, args.causal
        _, dev = make_attn_inputs(1, N, H_q, H_kv, d, 0, 1.0, device)
        out = torch.empty((1, N, H_q, d), dtype=torch.bfloat16, device=device)

        def fn():
            sqa.sqa_attn_fwd(dev["q"], dev["k"], dev["v"], out, 1, N, H_q, H_kv, d, causal, d ** -0.5, stream)
        for _ in range(args.warmup):
            fn()
        ms = _time_launches(fn, args.steps, flush, stream)
        assert sqa.sqa_device_status(stream) == 0
        fl = attn_flops(1, N, H_q, d, causal)
        med = statistics.median(ms)
        lines.append({"workload": "single", "N": N, "H_q": H_q, "H_kv": H_kv, "d": d, "causal": causal,
                      "ms_median": round(med, 3), "tflops": round(fl / (med * 1e-3) / 1e12, 1)})
        _emit(args, lines[-1])
    elif args.workload == "bwd":
        # attention backward (dq, dk, dv) at the forward's head configurations; --hq/--hkv/--d/--causal
        # given explicitly (hq != 16 or hkv != 16 or d != 64 or causal) time that one configuration instead
        import synth
        N = args.N
        if (args.hq, args.hkv, args.d, args.causal) != (16, 16, 64, 0):
            grid = [("single", args.hq, args.hkv, args.d, args.causal)]
        else:
            grid = [(n, hq, hkv, 64, 0) for n, hq, hkv in HEAD_CONFIGS_32K] + [("SQA-d128-causal", 16, 4, 128, 1)]
        for name, H_q, H_kv, d, causal in grid:
            _, dev = make_attn_inputs(1, N, H_q, H_kv, d, 0, 1.0, device)
            h = torch.empty((1, N, H_q, d), dtype=torch.bfloat16)
            synth.fill_bf16_into(h.data_ptr(), h.numel(), 0, "do", 1.0)
            do = h.to(device)
            out = torch.empty((1, N, H_q, d), dtype=torch.bfloat16, device=device)
            lse = torch.empty((1, H_q, N), dtype=torch.float32, device=device)
            sqa.sqa_attn_fwd_lse(dev["q"], dev["k"], dev["v"], out, lse, 1, N, H_q, H_kv, d, causal, d ** -0.5,
                                 stream)
            ws_bytes = sqa.sqa_attn_bwd_workspace_bytes(1, N, H_q)
            ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
            dq = torch.empty_like(out)
            dk = torch.empty_like(dev["k"])
            dv = torch.empty_like(dev["v"])

            def fn():
                sqa.sqa_attn_bwd(dev["q"], dev["k"], dev["v"], out, do, lse, dq, dk, dv, ws, ws_bytes, 1, N, H_q,
                                 H_kv, d, causal, d ** -0.5, stream)
            for _ in range(args.warmup):
                fn()
            ms = _time_launches(fn, args.steps, flush, stream)
            assert sqa.sqa_device_status(stream) == 0
            # algorithmic backward FLOPs: five N x N x d products per query head (S, dP, dV, dK, dQ)
            fl = 2.5 * attn_flops(1, N, H_q, d, causal)
            med = statistics.median(ms)
            lines.append({"workload": "bwd", "config": name, "N": N, "H_q": H_q, "H_kv": H_kv, "d": d,
                          "causal": causal, "ms_median": round(med, 3), "tflops": round(fl / (med * 1e-3) / 1e12, 1),
                          "pct_of_peak": round(100 * fl / (med * 1e-3) / 1e12 / peaks["bf16_tflops"], 1)})
            _emit(args, lines[-1])
            del dev, out, lse, ws, dq, dk, dv, do
    elif args.workload == "decode":
        # one new token per sequence against a 32768-token cache, the headline's head configurations;
        # memory-bound: bytes = the K/V cache (+ q and out), against the measured HBM copy bandwidth
        import synth
        B, N, d = args.B, args.N, args.d
        wanted = getattr(args, "decode_cfgs", None)
        for name, H_q, H_kv in HEAD_CONFIGS_32K:
            if wanted is not None and name not in wanted:
                continue

            def mk(shape, tensor):
                h = torch.empty(shape, dtype=torch.bfloat16)
                synth.fill_bf16_into(h.data_ptr(), h.numel(), 0, tensor, 1.0)
                return h.to(device)
            q, k, v = mk((B, H_q, d), "q"), mk((B, N, H_kv, d), "k"), mk((B, N, H_kv, d), "v")
            out = torch.empty((B, H_q, d), dtype=torch.bfloat16, device=device)
            ws_bytes = sqa.sqa_decode_workspace_bytes(B, N, H_q, H_kv, d)
            ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)

            def fn():
                sqa.sqa_decode_fwd(q, k, v, out, ws, ws_bytes, B, N, H_q, H_kv, d, d ** -0.5, stream)
            for _ in range(args.warmup):
                fn()
            ms = _time_launches(fn, args.steps, flush, stream, evict)
            assert sqa.sqa_device_status(stream) == 0
            med = statistics.median(ms)
            nbytes = 2.0 * B * N * H_kv * d * 2 + 2.0 * 2 * B * H_q * d
            gbs = nbytes / (med * 1e-3) / 1e9
            lines.append({"workload": "decode", "config": name, "B": B, "N": N, "H_q": H_q, "H_kv": H_kv, "d": d,
                          "us_median": round(med * 1e3, 2), "GB_per_s": round(gbs, 1),
                          "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 3), "bytes": int(nbytes)})
            _emit(args, lines[-1])
            del q, k, v, out, ws
    elif args.workload == "encoder":
        # encoder-style (non-causal) layer on one long sequence, the SQA abstract's compute-bound
        # scenario: x [1, N, 2048], d_head 64, per head configuration
        import synth
        B, N, dm, d = 1, args.N, 2048, 64

        def mk(shape, name, factor):
            h = torch.empty(shape, dtype=torch.bfloat16)
            synth.fill_bf16_into(h.data_ptr(), h.numel(), 0, name, factor)
            return h.to(device)
        x = mk((B, N, dm), "x", 1.0)
        out = torch.empty((B, N, dm), dtype=torch.bfloat16, device=device)
        for name, H_q, H_kv in (("MHA", 16, 16), ("GQA", 16, 4), ("SQA", 8, 4), ("xSQA", 4, 4)):
            wq, wk, wv = mk((H_q * d, dm), "wq", 0.02), mk((H_kv * d, dm), "wk", 0.02), mk((H_kv * d, dm), "wv", 0.02)
            wo = mk((dm, H_q * d), "wo", 0.02)
            ws_bytes = sqa.sqa_layer_workspace_bytes(B, N, dm, H_q, H_kv, d)
            ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)

            def fn():
                sqa.sqa_layer_fwd(x, wq, wk, wv, wo, out, ws, ws_bytes, B, N, dm, H_q, H_kv, d, 0, 0.125, stream)
            for _ in range(args.warmup):
                fn()
            ms = _time_launches(fn, args.steps, flush, stream)
            assert sqa.sqa_device_status(stream) == 0
            med = statistics.median(ms)
            fl_attn = attn_flops(B, N, H_q, d, False)
            fl_gemm = 2.0 * B * N * dm * (H_q + 2 * H_kv) * d + 2.0 * B * N * (H_q * d) * dm
            lines.append({"workload": "encoder", "config": name, "N": N, "H_q": H_q, "H_kv": H_kv, "d": d,
                          "d_model": dm, "ms_per_layer": round(med, 3),
                          "tflops_total": round((fl_attn + fl_gemm) / (med * 1e-3) / 1e12, 1)})
            _emit(args, lines[-1])
            del wq, wk, wv, wo, ws
    elif args.workload == "layer":
        import synth
        B, N, dm, H_q, H_kv, d = 4, 16384, 2048, 16, 8, 64
        M = B * N

        def mk(shape, name, factor):
            h = torch.empty(shape, dtype=torch.bfloat16)
            synth.fill_bf16_into(h.data_ptr(), h.numel(), 0, name, factor)
            return h.to(device)
        x = mk((B, N, dm), "x", 1.0)
        wq, wk, wv = mk((H_q * d, dm), "wq", 0.02), mk((H_kv * d, dm), "wk", 0.02), mk((H_kv * d, dm), "wv", 0.02)
        wo = mk((dm, H_q * d), "wo", 0.02)
        out = torch.empty((B, N, dm), dtype=torch.bfloat16, device=device)
        ws_bytes = sqa.sqa_layer_workspace_bytes(B, N, dm, H_q, H_kv, d)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)

        def fn():
            sqa.sqa_layer_fwd(x, wq, wk, wv, wo, out, ws, ws_bytes, B, N, dm, H_q, H_kv, d, 1, 0.125, stream)
        for _ in range(args.warmup):
            fn()
        ms = _time_launches(fn, args.steps, flush, stream)
        assert sqa.sqa_device_status(stream) == 0
        fl_attn = attn_flops(B, N, H_q, d, True)
        fl_gemm = 2.0 * M * dm * (H_q + 2 * H_kv) * d + 2.0 * M * (H_q * d) * dm
        med = statistics.median(ms)
        # per-kernel split
        qkv = torch.empty((M, (H_q + 2 * H_kv) * d), dtype=torch.bfloat16, device=device)
        wqkv = torch.cat([wq, wk, wv], 0).contiguous()
        ms_qkv = statistics.median(_time_launches(
            lambda: sqa.sqa_linear_fwd(x, wqkv, qkv, M, dm, (H_q + 2 * H_kv) * d, stream), args.steps, flush, stream))
        a = torch.empty((M, H_q * d), dtype=torch.bfloat16, device=device)
        ms_o = statistics.median(_time_launches(
            lambda: sqa.sqa_linear_fwd(a, wo, out, M, H_q * d, dm, stream), args.steps, flush, stream))
        lines.append({"workload": "layer", "ms_per_layer": round(med, 3), "tflops_total":
                      round((fl_attn + fl_gemm) / (med * 1e-3) / 1e12, 1), "ms_qkv_gemm": round(ms_qkv, 3),
                      "qkv_gemm_tflops": round(2.0 * M * dm * (H_q + 2 * H_kv) * d / (ms_qkv * 1e-3) / 1e12, 1),
                      "ms_o_gemm": round(ms_o, 3),
                      "o_gemm_tflops": round(2.0 * M * (H_q * d) * dm / (ms_o * 1e-3) / 1e12, 1),
                      "ms_attention_est": round(med - ms_qkv - ms_o, 3)})
        _emit(args, lines[-1])
    return lines


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["sqa", "reference"], default="sqa")
    ap.add_argument("--workload", choices=["headcfg32k", "small", "long", "layer", "sweep", "single", "linear", "bwd", "decode",
                             "encoder"],
                    default="headcfg32k")
    ap.add_argument("--N", type=int, default=32768)
    ap.add_argument("--B", type=int, default=8, help="sequences per decode step (--workload decode)")
    ap.add_argument("--hq", type=int, default=16)
    ap.add_argument("--hkv", type=int, default=16)
    ap.add_argument("--d", type=int, default=64)
    ap.add_argument("--causal", type=int, default=0)
    ap.add_argument("--M", type=int, default=65536)
    ap.add_argument("--K", type=int, default=2048)
    ap.add_argument("--N_out", type=int, default=2048)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="default workload: skip the extra measurements after the headline")
    ap.add_argument("--ingest-traffic", nargs="+", default=None, metavar="CSV",
                    help="write the per-launch DRAM traffic file from ncu CSV exports, then exit")
    args = ap.parse_args()
    if args.ingest_traffic:
        print(json.dumps(ingest_traffic(args.ingest_traffic)))
        return
    if args.warmup < 3 and args.impl == "sqa" and args.workload == "headcfg32k":
        print("note: raising --warmup to 3", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        r = bench_reference(args)
        if r is not None:
            print(json.dumps(r), flush=True)
        return
    if args.workload != "headcfg32k":
        bench_extra(args)
        return
    r = bench_sqa(args)
    if r is not None:
        print(json.dumps(r), flush=True)


if __name__ == "__main__":
    main()
