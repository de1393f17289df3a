"""The variants the pages leave open, through the C ABI against the oracle: a SwiGLU
MLP (the Qwen initialisation hint of the v0.1 blog's training Stage 1), a 3-D (t, y, x)
rotary embedding over the video raster, and 64-channel (2 x 2-patchified 16-channel)
latent tokens -- alone and together, at small shapes and at the 640x368 width, for a
solve and for the multi-unit pass.  Tolerances as elsewhere: relative L2 <= 1e-5 in
the fp32 mode, <= 2e-2 in bf16."""
import numpy as np
import pytest
import torch

import sfm_synth as S
from oracle import sfm_oracle as O
from tests._gpu_util import SMALL_BF16, ocfg, oracle_cache_layers, rel_l2, to_cuda, tol

pytestmark = pytest.mark.gpu

TINY3 = S.TINY.replace(grid_w=8)            # 8 x 8 video raster
SMALL3 = SMALL_BF16.replace(grid_w=20)      # 10 x 20 video raster

CASES = [
    TINY3.replace(name="tiny-swiglu", mlp="swiglu"),
    TINY3.replace(name="tiny-rope3d", rope="3d"),
    TINY3.replace(name="tiny-64ch", c_lat=64),
    TINY3.replace(name="tiny-all", mlp="swiglu", rope="3d", c_lat=64),
    SMALL3.replace(name="small-swiglu", mlp="swiglu"),
    SMALL3.replace(name="small-rope3d", rope="3d"),
    SMALL3.replace(name="small-64ch", c_lat=64),
    SMALL3.replace(name="small-all", mlp="swiglu", rope="3d", c_lat=64),
]


def _performer(w, weights, cache_units, max_sessions=1):
    from streaming_flow_matching_b200 import Performer
    pool = max_sessions * (cache_units * w.unit_kv_tokens + w.n_tokens)
    return Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=max_sessions)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_variant_step_and_solve_match_oracle(cuda_device, w):
    weights_cpu = S.make_weights(w)
    n_units = w.cache_units + 2                     # the ring has wrapped: t and p0 keep counting
    k, v = S.make_kv_slices(w, n_units)
    p = _performer(w, to_cuda(weights_cpu), w.cache_units)
    s = p.open_session(w.cache_units)
    p.kvcache_append(s, k.cuda(), v.cuda())
    ck, cv = oracle_cache_layers(k, v, n_units, w.unit_kv_tokens, w.cache_units)
    valid, p0 = w.cache_units * w.unit_kv_tokens, n_units * w.unit_kv_tokens
    _, eps = S.make_latents(w)
    eps = eps[0]
    taus = S.uniform_taus(w.n_steps)
    z = eps.cuda().clone()
    vel = torch.empty_like(z)
    p.denoise_step(s, z, taus[0], taus[1], vel)
    torch.cuda.synchronize()
    ref_v = O.f_theta(ocfg(w), eps, taus[0], weights_cpu, ck, cv, valid, p0)
    e_v = rel_l2(vel.cpu().numpy(), ref_v)
    z = eps.cuda().clone()
    p.fm_solve(s, z, taus)
    torch.cuda.synchronize()
    ref_z = O.denoise_solve(ocfg(w), eps, taus, weights_cpu, ck, cv, valid, p0)
    e_z = rel_l2(z.cpu().numpy(), ref_z)
    print(f"{w.name}: velocity {e_v:.3e}  solve {e_z:.3e}")
    assert p.check_device_error() == 0
    assert e_v <= tol(w) and e_z <= tol(w)
    p.close()


def test_variants_at_640x368_width_match_oracle(cuda_device):
    # SwiGLU (W_1 [24576][3072]), 3-D RoPE over the 23 x 40 raster, 64-channel tokens;
    # 2 layers over a 12-unit cache
    w = S.V02.replace(name="v0.2-variants", n_layers=2, cache_units=12, mlp="swiglu", rope="3d",
                      grid_w=40, c_lat=64)
    weights_cpu = S.make_weights(w)
    k, v = S.make_kv_slices(w, w.cache_units)
    p = _performer(w, to_cuda(weights_cpu), w.cache_units)
    s = p.open_session(w.cache_units)
    p.kvcache_append(s, k.cuda(), v.cuda())
    _, eps = S.make_latents(w)
    z = eps[0].cuda().clone()
    vel = torch.empty_like(z)
    p.denoise_step(s, z, 0.75, 0.5, vel)
    torch.cuda.synchronize()
    valid = w.cache_units * w.unit_kv_tokens
    ref = O.f_theta(ocfg(w), eps[0], 0.75, weights_cpu, list(k), list(v), valid, valid)
    e = rel_l2(vel.cpu().numpy(), ref)
    print(f"640x368 width, SwiGLU + 3-D RoPE + 64 channels: velocity {e:.3e}")
    assert p.check_device_error() == 0 and e <= tol(w)
    p.close()


@pytest.mark.parametrize("w", [CASES[3], CASES[7]], ids=lambda w: w.name)
def test_variant_units_pass_matches_oracle(cuda_device, w):
    # several units in one pass: with 3-D RoPE every unit takes the next time index
    n_units, cu = 3, 10
    weights_cpu = S.make_weights(w)
    p = _performer(w, to_cuda(weights_cpu), cu, n_units)
    s = p.open_session(cu)
    k, v = S.make_kv_slices(w, 2)
    p.kvcache_append(s, k.cuda(), v.cuda())
    ck, cv = oracle_cache_layers(k, v, 2, w.unit_kv_tokens, cu)
    g = torch.Generator().manual_seed(63)
    zs = [torch.randn(w.n_tokens, w.c_lat, generator=g) for _ in range(n_units)]
    taus = [0.0, 0.4, 1.0]
    vel = p.velocity_units(s, [z.cuda() for z in zs], taus)
    torch.cuda.synchronize()
    valid = 2 * w.unit_kv_tokens
    ref = O.f_theta_units(ocfg(w), zs, taus, weights_cpu, ck, cv, valid, valid)
    for u in range(n_units):
        e = rel_l2(vel[u].cpu().numpy(), ref[u])
        print(f"{w.name} unit {u}: rel L2 {e:.3e}")
        assert e <= tol(w)
    p.close()
