"""Micro-benchmarks of single kernels of the hot path, timed with CUDA events.

  python -m streaming_flow_matching_b200.microbench attention --n-kv 16800 [--n-q 924 --heads 24]
  python -m streaming_flow_matching_b200.microbench attention --n-q 3696 --n-kv 61296 --unit-tokens 924
  python -m streaming_flow_matching_b200.microbench append [--layers 28 --units 1]
  python -m streaming_flow_matching_b200.microbench euler [--n 268435456]
  python -m streaming_flow_matching_b200.microbench linear --m 924 --n 12288 --k 3072 [--epilogue gelu]
  python -m streaming_flow_matching_b200.microbench step [--layers 1 --cache-units 4]
  python -m streaming_flow_matching_b200.microbench guided --cache-units 48 [--steps 4 --scale 5]
  python -m streaming_flow_matching_b200.microbench sweep      # attention + append sweep

Inputs are seeded and larger than L2 where the case allows; each timing is
the median of --reps launches after --warmup launches.  Prints one JSON line
per case.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import sfm_synth as S  # noqa: E402
from streaming_flow_matching_b200 import (Performer, attention, attention_workspace_bytes,  # noqa: E402
                                          euler_update, linear)


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def _time(fn, warmup, reps):
    """Median of `reps` single calls, each bracketed by events (host work of the call
    included when the GPU waits for it)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def _time_b2b(fn, reps):
    """Mean device time per call over `reps` calls enqueued back to back (the host runs
    ahead of the GPU, so gaps between launches vanish unless a call's host work is
    longer than its kernels)."""
    fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    b.synchronize()
    return a.elapsed_time(b) / reps


def bench_attention(n_q, n_kv, heads, warmup, reps, unit=None):
    """unit: None for every key visible; else block-causal over query units of `unit`
    tokens (the first n_kv - n_q keys a shared prefix).  FLOPs count the visible
    keys only: 4 D H per (query, visible key)."""
    q, k, v = S.make_qkv(n_q, n_kv, heads, 128, device="cuda")
    o = torch.empty_like(q)
    ws_n = attention_workspace_bytes(n_q, n_kv, heads, 128)
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device="cuda")
    call = lambda: attention(q, k, v, o, ws, unit_tokens=unit)  # noqa: E731
    ms_single = _time(call, warmup, reps)
    ms = _time_b2b(call, max(reps, 20))
    if unit is None:
        visible = n_q * n_kv
    else:
        prefix = n_kv - n_q
        visible = sum(prefix + min((i // unit + 1) * unit, n_q) for i in range(n_q))
    flop = 4.0 * visible * heads * 128
    hbm, bf16, src = _peaks()
    tf = flop / (ms / 1e3) / 1e12
    out = {"case": "attention", "n_q": n_q, "n_kv": n_kv, "heads": heads, "ms": ms,
           "ms_single_call": ms_single, "tflops": tf, "frac_of_bf16_burst": tf / bf16,
           "peak_source": src, "timing": "ms: back-to-back mean; ms_single_call: median"}
    if unit is not None:
        out.update({"unit_tokens": unit, "visible_fraction": visible / (n_q * n_kv)})
    return out


def bench_append(layers, units, warmup, reps):
    w = S.V02.replace(n_layers=layers)
    p = Performer.from_workload(w, None)
    s = p.open_session(w.cache_units)
    g = torch.Generator(device="cuda")
    g.manual_seed(2)
    shape = (layers, units * w.unit_kv_tokens, w.n_heads, w.head_dim)
    k = torch.randn(*shape, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(*shape, generator=g, device="cuda").to(torch.bfloat16)
    ms = _time(lambda: p.kvcache_append(s, k, v), warmup, reps)
    nbytes = 2 * 2 * k.numel() * 2
    hbm, _, src = _peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    p.close()
    return {"case": "append", "layers": layers, "units": units, "bytes": nbytes, "ms": ms,
            "gb_s": gbs, "frac_of_hbm": gbs / hbm, "peak_source": src}


def bench_linear(m, n, k, epilogue, warmup, reps):
    g = torch.Generator(device="cuda")
    g.manual_seed(6)
    x = torch.randn(m, k, generator=g, device="cuda").to(torch.bfloat16)
    w = (0.02 * torch.randn(n, k, generator=g, device="cuda")).to(torch.bfloat16)
    y = torch.zeros(m, n, device="cuda",
                    dtype=torch.bfloat16 if epilogue in ("out", "gelu") else torch.float32)
    ms = _time(lambda: linear(x, w, y, epilogue), warmup, reps)
    _, bf16, src = _peaks()
    tf = 2.0 * m * n * k / (ms / 1e3) / 1e12
    return {"case": "linear", "m": m, "n": n, "k": k, "epilogue": epilogue, "ms": ms,
            "tflops": tf, "frac_of_bf16_burst": tf / bf16, "peak_source": src}


def bench_euler(n, warmup, reps):
    g = torch.Generator(device="cuda")
    g.manual_seed(4)
    z = torch.randn(n, generator=g, device="cuda")
    v = torch.randn(n, generator=g, device="cuda")
    ms = _time(lambda: euler_update(z, v, -0.25), warmup, reps)
    hbm, _, src = _peaks()
    gbs = 12.0 * n / (ms / 1e3) / 1e9
    return {"case": "euler", "n": n, "ms": ms, "gb_s": gbs, "frac_of_hbm": gbs / hbm,
            "peak_source": src}


def bench_step(layers, cache_units, warmup, reps):
    """One Euler step (denoise_step) at the 640x368 unit width with `layers` layers and a
    `cache_units`-unit cache: a small-memory stand-in for ncu captures of the step's kernels."""
    w = S.V02.replace(name=f"v0.2-width-{layers}L", n_layers=layers, cache_units=cache_units)
    dev = torch.device("cuda", 0)
    weights = S.make_weights(w, device=dev)
    pool = cache_units * w.unit_kv_tokens + w.n_tokens
    p = Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=1)
    s_id = p.open_session(cache_units)
    k, v = S.make_kv_slices(w, cache_units, device=dev)
    p.kvcache_append(s_id, k, v)
    _, eps = S.make_latents(w, device=dev)
    z = eps[0].clone()
    ms = _time(lambda: p.denoise_step(s_id, z, 1.0, 0.75), warmup, reps)
    p.check_device_error()
    return {"case": "step", "layers": layers, "cache_tokens": cache_units * w.unit_kv_tokens,
            "ms": ms}


def bench_guided(layers, cache_units, n_steps, scale, warmup, reps):
    """Classifier-free-guided solve at the 640x368 unit (conditional session with a full
    cache_units-unit cache, unconditional session with an empty cache) next to the plain
    solve of the same session: both timed as whole solves of n_steps Euler steps."""
    w = S.V02.replace(name=f"v0.2-{layers}L", n_layers=layers, cache_units=cache_units)
    dev = torch.device("cuda", 0)
    weights = S.make_weights(w, device=dev)
    pool = cache_units * w.unit_kv_tokens + w.n_tokens + w.unit_kv_tokens + w.n_tokens
    p = Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=2)
    s_id = p.open_session(cache_units)
    u_id = p.open_session(1)
    k, v = S.make_kv_slices(w, cache_units, device=dev)
    p.kvcache_append(s_id, k, v)
    del k, v
    _, eps = S.make_latents(w, device=dev)
    taus = S.uniform_taus(n_steps)
    z = eps[0].clone()

    def plain():
        z.copy_(eps[0])
        p.fm_solve(s_id, z, taus)

    def guided():
        z.copy_(eps[0])
        p.fm_solve_guided(s_id, u_id, z, taus, scale)

    ms_plain = _time(plain, warmup, reps)
    ms_guided = _time(guided, warmup, reps)
    p.check_device_error()
    return {"case": "guided", "layers": layers, "cache_tokens": cache_units * w.unit_kv_tokens,
            "steps": n_steps, "scale": scale, "ms_guided_solve": ms_guided,
            "ms_plain_solve": ms_plain, "guided_over_plain": ms_guided / ms_plain,
            "guided_steps_per_s": n_steps / ms_guided * 1e3}


def bench_units(layers, cache_units, n_units, warmup, reps):
    """A multi-unit pass (sfm_velocity_units) at the 640x368 unit: n_units units after a
    cache_units-unit cache (0: a scene's first pass), all at tau = 0, 28 layers by default."""
    w = S.V02.replace(name=f"v0.2-{layers}L", n_layers=layers, cache_units=max(cache_units, 1))
    dev = torch.device("cuda", 0)
    weights = S.make_weights(w, device=dev)
    cap = max(cache_units + n_units, 1)
    pool = cap * w.unit_kv_tokens + w.n_tokens
    p = Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=n_units)
    s_id = p.open_session(cap)
    if cache_units:
        k, v = S.make_kv_slices(w, cache_units, device=dev)
        p.kvcache_append(s_id, k, v)
        del k, v
    g = torch.Generator(device=dev)
    g.manual_seed(61)
    zs = [torch.randn(w.n_tokens, w.c_lat, generator=g, device=dev) for _ in range(n_units)]
    vs = [torch.empty_like(z) for z in zs]
    taus = [0.0] * n_units
    ms = _time(lambda: p.velocity_units(s_id, zs, taus, v_outs=vs), warmup, reps)
    p.check_device_error()
    n = w.n_tokens
    valid = cache_units * w.unit_kv_tokens
    # visible keys: the cache plus the units up to each query's own
    attn = sum(4 * n * (valid + (u + 1) * n) * w.hd for u in range(n_units))
    gemm = n_units * (2 * n * w.d_model * 3 * w.hd + 2 * n * w.hd * w.d_model + 4 * n * w.d_model * w.d_mlp)
    flop = layers * (attn + gemm)
    return {"case": "units", "layers": layers, "units": n_units, "cache_tokens": valid,
            "ms": ms, "tflops": flop / (ms / 1e3) / 1e12}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["attention", "append", "euler", "linear", "step", "guided",
                                    "units", "sweep"])
    ap.add_argument("--cache-units", type=int, default=4)
    ap.add_argument("--m", type=int, default=924)
    ap.add_argument("--k", type=int, default=3072)
    ap.add_argument("--epilogue", default="gelu")
    ap.add_argument("--n-q", type=int, default=924)
    ap.add_argument("--n-kv", type=int, default=57600 + 924)
    ap.add_argument("--heads", type=int, default=24)
    ap.add_argument("--unit-tokens", type=int, default=None,
                    help="attention: block-causal over query units of this many tokens")
    ap.add_argument("--layers", type=int, default=28)
    ap.add_argument("--units", type=int, default=1)
    ap.add_argument("--n", type=int, default=1 << 28)
    ap.add_argument("--steps", type=int, default=4)
    ap.add_argument("--scale", type=float, default=5.0)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--reps", type=int, default=10)
    a = ap.parse_args()
    torch.cuda.set_device(0)
    out = []
    if a.case == "attention":
        out.append(bench_attention(a.n_q, a.n_kv, a.heads, a.warmup, a.reps, a.unit_tokens))
    elif a.case == "append":
        out.append(bench_append(a.layers, a.units, a.warmup, a.reps))
    elif a.case == "euler":
        out.append(bench_euler(a.n, a.warmup, a.reps))
    elif a.case == "linear":
        out.append(bench_linear(a.m, a.n, a.k, a.epilogue, a.warmup, a.reps))
    elif a.case == "step":
        out.append(bench_step(a.layers, a.cache_units, a.warmup, a.reps))
    elif a.case == "guided":
        out.append(bench_guided(a.layers, a.cache_units, a.steps, a.scale, a.warmup, a.reps))
    elif a.case == "units":
        out.append(bench_units(a.layers, a.cache_units, a.units, a.warmup, a.reps))
    else:
        for m, n, k, e in [(924, 9216, 3072, "f32"), (924, 3072, 3072, "resid"),
                           (924, 12288, 3072, "gelu"), (924, 3072, 12288, "resid")]:
            out.append(bench_linear(m, n, k, e, a.warmup, a.reps))
        for n_kv in S.ATTN_SWEEP_TOKENS:
            out.append(bench_attention(a.n_q, n_kv + a.n_q, a.heads, a.warmup, a.reps))
        out.append(bench_append(1, 1, a.warmup, a.reps))
        out.append(bench_append(a.layers, 1, a.warmup, a.reps))
        out.append(bench_euler(a.n, a.warmup, a.reps))
    for o in out:
        print(json.dumps(o), flush=True)


if __name__ == "__main__":
    main()
