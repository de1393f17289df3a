#!/usr/bin/env python
"""Benchmark: the performer's next-unit denoise of a 640x368 unit on B200.

One bench step = one pass of the whole hot path for one unit: the thinker's
1200-token K/V slice is appended to the session's 48-unit ring cache (evicting
the oldest unit, so 57,600 cached tokens stay valid), then the 924 latent
tokens (920 video + 4 audio) are solved from noise with 4 Euler steps of the
28-layer velocity network.  Inputs are synthetic (seeded), resident in HBM and
far larger than L2 (6.3 GB of weights + 19.8 GB of cache are read per Euler
step), so no L2 flush is needed between steps.

value = Euler denoise steps per second summed over all ranks (each rank runs
its own session: weak scaling, no collective on the data path), timed over K
steps of the product path (each solve is one captured CUDA graph).  The
per-kernel device times (kernel_ms_per_unit, roofline, contractions) come from
a second pass of the same K steps with CUDA events around every launch.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "640x368 unit denoise steps/s"
UNIT = "denoise steps/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="v0.2-640x368")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16": p["bf16_tflops"],
                "bf16_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        cmd = ["nvidia-smi", f"--id={self.index}", "--query-gpu=" + ",".join(self.FIELDS),
               "--format=csv,noheader,nounits", "-lms", "200"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, val in zip(names, parts[3:]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# multi-rank aggregation (one session per rank, no collective on the data path)
# ---------------------------------------------------------------------------
def max_over_ranks(ms, device=None):
    """Largest per-rank device time of the timed region (every rank calls this)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def whole_job_rate(n_units_per_rank, euler_steps, world, ms_max):
    """Euler denoise steps per second summed over all ranks (weak scaling: each rank
    solves its own units), timed by the slowest rank."""
    return euler_steps * n_units_per_rank * world / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# work counts
# ---------------------------------------------------------------------------
def flop_counts(w, valids):
    """valids: valid cached tokens of each session of the batch."""
    n, d, hd, f, L = w.n_tokens, w.d_model, w.hd, w.d_mlp, w.n_layers
    attn = sum(4 * n * (valid + n) * hd for valid in valids)
    gemm = len(valids) * (2 * n * d * 3 * hd + 2 * n * hd * d + 2 * n * d * f + 2 * n * f * d)
    return {"attention_per_launch": attn, "gemm_per_layer": gemm,
            "per_euler_step": L * (attn + gemm)}


def gemm_flops_per_layer(w, n_sessions):
    """2 M K N of each projection of one layer (M = sessions x unit tokens)."""
    m, d, hd, f = n_sessions * w.n_tokens, w.d_model, w.hd, w.d_mlp
    return {"gemm_qkv": 2 * m * d * 3 * hd, "gemm_o": 2 * m * hd * d,
            "gemm_up": 2 * m * d * f, "gemm_down": 2 * m * f * d}


def append_bytes(w):
    return 2 * 2 * w.n_layers * w.unit_kv_tokens * w.hd * 2   # K and V, read + write, bf16


KERNEL_END = b"}  // namespace atc\n"   # the attention source's device code ends here


def kernel_hash(path):
    """sha256 (16 hex digits) of a kernel source's device code: the text up to the end of
    its kernel namespace (host-side launch and planning code after it does not change the
    kernel's memory traffic)."""
    with open(path, "rb") as f:
        src = f.read()
    end = src.find(KERNEL_END)
    return hashlib.sha256(src if end < 0 else src[:end + len(KERNEL_END)]).hexdigest()[:16]


def traffic_for(kernel_src, table=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this kernel
    code; None otherwise."""
    path = table or os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        ent = t[os.path.basename(kernel_src)]
        if ent["kernel_sha256_16"] != kernel_hash(kernel_src):
            return None
        return ent["dram_bytes_per_launch"]
    except Exception:
        return None


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the same workload
# ---------------------------------------------------------------------------
# layers of f_theta the CPU baseline times (both arms): each runs over the full cache
CPU_SAMPLE_LAYERS = 1
# datasheet figures of a B200, for context next to the measured denominators
DATASHEET = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def cpu_sample(w, n_layers=CPU_SAMPLE_LAYERS):
    """Time the oracle's f_theta at the bench shapes on a bounded sample: the
    embedding, n_layers of the 28 layers (each over the full 57,600-token cache),
    and the head; extrapolate to one Euler step.  Returns (seconds per Euler step,
    description): the sample is extrapolated, never a full step."""
    import numpy as np
    import torch
    from threadpoolctl import threadpool_info

    import sfm_synth as S
    from oracle import sfm_oracle as O

    cfg = O.Config(w.n_layers, w.d_model, w.n_heads, w.head_dim, w.d_mlp, w.c_lat, w.n_video,
                   w.n_audio, w.unit_kv_tokens, w.rope_theta, w.rms_eps)
    one = w.replace(n_layers=1)
    weights = S.make_weights(one)
    k, v = S.make_kv_slices(one, w.cache_units)
    _, eps = S.make_latents(w)
    valid = w.cache_units * w.unit_kv_tokens
    kc, vc = O.f64(k[0]), O.f64(v[0])
    lw = {n: O.f64(t) for n, t in weights["layers"][0].items()}
    t0 = time.perf_counter()
    x = O.embed(cfg, eps[0], 1.0, weights)
    t_embed = time.perf_counter() - t0
    pos = valid + np.arange(w.n_tokens)
    layer_times = []
    for _ in range(n_layers):
        t0 = time.perf_counter()
        x = O.layer_forward(cfg, x, lw, kc, vc, pos)
        layer_times.append(time.perf_counter() - t0)
    t0 = time.perf_counter()
    O.head(cfg, x, weights)
    t_head = time.perf_counter() - t0
    measured = t_embed + sum(layer_times) + t_head
    t_step = t_embed + w.n_layers * statistics.mean(layer_times) + t_head
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    info = {"cores": os.cpu_count(), "threads": threads, "timed_layers": len(layer_times),
            "extrapolated": True, "measured_s": measured,
            "sample": (f"oracle f_theta (numpy fp64) at the {w.name} unit over the full "
                       f"{valid}-token cache: embed + {len(layer_times)} of {w.n_layers} layers "
                       f"+ head timed, x{w.n_layers}/{len(layer_times)} layers extrapolated to "
                       "one Euler step")}
    del torch
    return t_step, info


def run_reference(args, w):
    """The oracle as the reference arm: each of the K steps times one bounded sample
    (embedding + CPU_SAMPLE_LAYERS layers over the full cache + head) and extrapolates
    it to one Euler step; ms_per_step is that extrapolation x the unit's Euler steps,
    and measured_wall_s the wall time the timed samples actually took."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    for _ in range(args.warmup):
        cpu_sample(w)
    times = []
    wall0 = time.perf_counter()
    for _ in range(args.steps):
        t, info = cpu_sample(w)
        times.append(t)
    wall = time.perf_counter() - wall0
    t_step = statistics.mean(times)
    value = 1.0 / t_step
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_step * 1e3 * w.n_steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": config_of(w),
            "extrapolated": True, "timed_layers": info["timed_layers"],
            "measured_wall_s": wall,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": info["cores"],
                             "threads": info["threads"], "kind": "oracle",
                             "timed_layers": info["timed_layers"], "extrapolated": True,
                             "sample": info["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def session_caps(w):
    """Cache capacity (units) of each session the workload runs."""
    import sfm_synth as S
    if w.name == S.V02X8.name:
        return S.session_cache_units(unit_tokens=w.unit_kv_tokens)
    return [w.cache_units]


def config_of(w):
    caps = session_caps(w)
    cfg = {"workload": f"{w.name} unit: kvcache_append of one {w.unit_kv_tokens}-token slice + "
                       f"{w.n_steps}-step Euler solve",
           "sessions": len(caps), "tokens_per_unit": w.n_tokens, "video_tokens": w.n_video,
           "audio_tokens": w.n_audio, "layers": w.n_layers,
           "d_model": w.d_model, "heads": w.n_heads, "head_dim": w.head_dim, "d_mlp": w.d_mlp,
           "euler_steps": w.n_steps,
           "l2": "inputs larger than L2 (weights + cache read every Euler step)"}
    if len(caps) == 1:
        cfg["cache_tokens"] = caps[0] * w.unit_kv_tokens
        cfg["parallelism"] = "one session per GPU, no collectives"
    else:
        cfg["cache_tokens"] = [c * w.unit_kv_tokens for c in caps]
        cfg["parallelism"] = (f"{len(caps)} sessions batched per GPU (ragged caches, varlen "
                              "attention), no collectives")
    return cfg


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import sfm_synth as S
    from streaming_flow_matching_b200 import Performer, _lib as L

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    weights = S.make_weights(w, device=dev)
    caps = session_caps(w)
    n_sess = len(caps)
    pool = sum(c * w.unit_kv_tokens + w.n_tokens for c in caps)
    p = Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=n_sess)
    sessions = []
    for i, cap in enumerate(caps):
        s_id = p.open_session(cap)
        k, v = S.make_kv_slices(w.replace(cache_units=cap), cap, device=dev, seed=S.SEED_CACHE + 10 * i)
        p.kvcache_append(s_id, k, v)
        del k, v
        sessions.append(s_id)
    g = torch.Generator(device=dev)
    g.manual_seed(11 + rank)
    shape = (w.n_layers, w.unit_kv_tokens, w.n_heads, w.head_dim)
    k1 = torch.randn(*shape, generator=g, device=dev).to(torch.bfloat16)
    v1 = torch.randn(*shape, generator=g, device=dev).to(torch.bfloat16)
    _, eps = S.make_latents(w, device=dev, n_sessions=n_sess)
    zs = [eps[i].clone() for i in range(n_sess)]
    taus = S.uniform_taus(w.n_steps)
    torch.cuda.synchronize()

    def solve_all():
        if n_sess == 1:
            p.fm_solve(sessions[0], zs[0], taus)
        else:
            p.fm_solve_batched(sessions, zs, taus)

    def step():
        for s_id in sessions:
            p.kvcache_append(s_id, k1, v1)
        for i in range(n_sess):
            zs[i].copy_(eps[i])
        solve_all()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.4)
    # the timed region: the product path (each solve one captured CUDA graph)
    n0 = L.lib.sfm_kernel_launch_count()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = L.lib.sfm_kernel_launch_count() - n0
    clocks = sampler.stop()
    ms_max = max_over_ranks(e0.elapsed_time(e1), dev)
    barrier()

    # per-kernel device times: the same K steps again with a CUDA event pair around
    # every launch, on the launching stream (the library then launches directly:
    # event pairs inside the graph would perturb the timed region above)
    torch.cuda.synchronize()
    L.profile_begin(1 << 16)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    prof = L.profile_end()
    prof_ms_max = max_over_ranks(e0.elapsed_time(e1), dev)
    barrier()

    # end to end: host (pinned) inputs copied in and the latents copied out every step.
    # As in a streaming performer, the next unit's K/V slice is copied into a second
    # device staging buffer on a copy stream while the current unit is solved; the
    # append itself waits for the solve (it overwrites the oldest ring slot, which the
    # solve reads).  The latents' ε in and z out are copied on the compute stream.
    e2e = None
    if not args.no_e2e:
        k1_h = k1.cpu().pin_memory()
        v1_h = v1.cpu().pin_memory()
        eps_h = [eps[i].cpu().pin_memory() for i in range(n_sess)]
        z_h = [torch.empty_like(e).pin_memory() for e in eps_h]
        stage = [[(torch.empty_like(k1), torch.empty_like(v1)) for _ in sessions] for _ in range(2)]
        copy_stream = torch.cuda.Stream(device=dev)
        landed = [torch.cuda.Event() for _ in range(2)]
        consumed = [torch.cuda.Event() for _ in range(2)]

        def copy_in(buf):
            # every session receives its own slice from host memory
            copy_stream.wait_event(consumed[buf])
            with torch.cuda.stream(copy_stream):
                for kb, vb in stage[buf]:
                    kb.copy_(k1_h, non_blocking=True)
                    vb.copy_(v1_h, non_blocking=True)
            landed[buf].record(copy_stream)

        def e2e_step(i):
            cur = i & 1
            stream.wait_event(landed[cur])
            for s_id, (kb, vb) in zip(sessions, stage[cur]):
                p.kvcache_append(s_id, kb, vb)
            consumed[cur].record(stream)
            copy_in(cur ^ 1)                       # the next unit's slices, during this solve
            for i2 in range(n_sess):
                zs[i2].copy_(eps_h[i2], non_blocking=True)
            solve_all()
            for i2 in range(n_sess):
                z_h[i2].copy_(zs[i2], non_blocking=True)

        for e in consumed:
            e.record(stream)
        n_warm = max(1, args.warmup)
        copy_in(0)
        for i in range(n_warm):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for i in range(n_warm, n_warm + args.steps):
            e2e_step(i)
        stream.wait_event(landed[(n_warm + args.steps) & 1])   # the last copy, too
        e1.record(stream)
        torch.cuda.synchronize()
        te_max = max_over_ranks(e0.elapsed_time(e1), dev)
        h2d = n_sess * (k1.numel() * 2 + v1.numel() * 2 + eps[0].numel() * 4)
        e2e = {"value": whole_job_rate(args.steps * n_sess, w.n_steps, world, te_max), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": n_sess * eps[0].numel() * 4,
               "overlap": "the next unit's K/V slices are copied to the device during the current solve"}
        barrier()

    if rank == 0:
        pk = peaks()
        fl = flop_counts(w, [c * w.unit_kv_tokens for c in caps])
        a_ms, a_n = prof["attention"]
        attn_avg_ms = a_ms / max(a_n, 1)
        attn_tflops = fl["attention_per_launch"] / (attn_avg_ms / 1e3) / 1e12
        gemm_ms = sum(prof[k][0] for k in ("gemm_qkv", "gemm_o", "gemm_up", "gemm_down"))
        contraction_ms = a_ms + prof["attention_merge"][0] + gemm_ms
        contraction_flop = args.steps * w.n_steps * fl["per_euler_step"]
        contr_tflops = contraction_flop / (contraction_ms / 1e3) / 1e12
        # each projection against the measured peaks (2 M K N per launch, L launches per step)
        gemm_fracs = {}
        for key, flop in gemm_flops_per_layer(w, len(caps)).items():
            ms_k = prof[key][0]
            if ms_k > 0:
                tf = args.steps * w.n_steps * w.n_layers * flop / (ms_k / 1e3) / 1e12
                gemm_fracs[key] = {"tflops": tf, "frac": tf / pk["bf16_sustained"],
                                   "frac_of_burst": tf / pk["bf16"],
                                   "ms_per_unit": ms_k / args.steps}
        ap_ms, ap_n = prof["append"]
        append_gbs = append_bytes(w) / (ap_ms / max(ap_n, 1) / 1e3) / 1e9 if ap_n else None
        unit_ms = ms_max / args.steps
        attn_src = os.path.join(ROOT, "streaming_flow_matching_b200", "csrc", "attn_tc.cu")
        traffic = traffic_for(attn_src)
        line = {
            "metric": METRIC,
            "value": whole_job_rate(args.steps * n_sess, w.n_steps, world, ms_max),
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": unit_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded), resident in HBM",
            "config": config_of(w),
            "unit_latency_ms": unit_ms,
            "e2e": e2e,
            "gpu_launches": launches,
            "roofline": {"kernel": "attn_tc_kernel (tcgen05 flash attention, split-KV)", "bound": "tensor",
                         "achieved": attn_tflops, "peak": pk["bf16_sustained"],
                         "unit": "TFLOP/s", "frac": attn_tflops / pk["bf16_sustained"],
                         "frac_of_burst": attn_tflops / pk["bf16"],
                         "frac_of_datasheet": attn_tflops / DATASHEET["bf16_tflops"],
                         "traffic": traffic,
                         "peak_note": f"{pk['source']} sustained bf16 (kernel timed inside a long step)",
                         "flop_per_launch": fl["attention_per_launch"],
                         "avg_launch_ms": attn_avg_ms,
                         "timing": "CUDA events around each launch on its stream, over a second "
                                   "timed pass of the same steps (direct launches)"},
            "contractions": {"tflops": contr_tflops,
                             "frac_of_bf16_peak": contr_tflops / pk["bf16_sustained"],
                             "frac_of_burst": contr_tflops / pk["bf16"],
                             "frac_of_datasheet": contr_tflops / DATASHEET["bf16_tflops"],
                             "projections": gemm_fracs,
                             "attn_gemm_device_ms_per_unit": contraction_ms / args.steps},
            "append": {"gb_s": append_gbs, "frac_of_hbm": (append_gbs / pk["hbm_gbs"]) if append_gbs else None,
                       "frac_of_datasheet": (append_gbs / DATASHEET["hbm_gbs"]) if append_gbs else None,
                       "bytes": append_bytes(w)},
            "peaks": {"bf16_sustained_tflops": pk["bf16_sustained"], "bf16_burst_tflops": pk["bf16"],
                      "hbm_gbs": pk["hbm_gbs"], "source": pk["source"],
                      "datasheet_bf16_tflops": DATASHEET["bf16_tflops"],
                      "datasheet_hbm_gbs": DATASHEET["hbm_gbs"]},
            "kernel_ms_per_unit": {k2: round(v2[0] / args.steps, 4) for k2, v2 in prof.items()},
            "profiled_pass_ms_per_step": prof_ms_max / args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline and n_sess == 1:
            t_step, info = cpu_sample(w)
            line["cpu_baseline"] = {"value": 1.0 / t_step, "unit": UNIT, "cores": info["cores"],
                                    "threads": info["threads"], "kind": "oracle",
                                    "timed_layers": info["timed_layers"], "extrapolated": True,
                                    "measured_s": info["measured_s"], "sample": info["sample"]}
        print(json.dumps(line), flush=True)
    p.close()
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    import sfm_synth as S
    w = S.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
