"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Sizes: the tiny fp32 and small bf16 cases span several tiles with ragged
tails and run the oracle in seconds; the 192x336 (28 layers) and 640x368
(full width, full 57,600-token cache) cases compare a whole denoise step with
the oracle.  Tolerances: cache contents bit-exact; relative L2 <= 2e-2 for
bf16 velocities and latents, <= 1e-5 in the fp32 mode.
"""
import numpy as np
import pytest
import torch

import sfm_synth as S
from oracle import sfm_oracle as O
from tests._gpu_util import (BF16_TOL, FP32_TOL, SMALL_BF16, WIDE_BF16, ocfg, oracle_cache_layers,
                             rel_l2, to_cuda, tol)

pytestmark = pytest.mark.gpu


def _performer(w, weights, cache_units=None, extra_sessions=0, ring=True):
    from streaming_flow_matching_b200 import Performer
    cu = cache_units or w.cache_units
    pool = (1 + extra_sessions) * (cu * w.unit_kv_tokens + w.n_tokens)
    return Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=1 + extra_sessions,
                                   ring=ring)


def _setup(w, n_units=None, cache_units=None):
    """Weights, slices, a performer with one session holding n_units units."""
    n_units = w.cache_units if n_units is None else n_units
    cache_units = cache_units or w.cache_units
    weights_cpu = S.make_weights(w)
    weights = to_cuda(weights_cpu)
    k, v = S.make_kv_slices(w, n_units)
    p = _performer(w, weights, cache_units)
    s = p.open_session(cache_units)
    p.kvcache_append(s, k.cuda(), v.cuda())
    return weights_cpu, weights, k, v, p, s


def _oracle_velocity(w, weights_cpu, k, v, n_units, eps, tau):
    ck, cv = oracle_cache_layers(k, v, n_units, w.unit_kv_tokens, w.cache_units)
    valid = min(n_units, w.cache_units) * w.unit_kv_tokens
    return O.f_theta(ocfg(w), eps, tau, weights_cpu, ck, cv, valid, n_units * w.unit_kv_tokens)


# ---------------------------------------------------------------------------
# whole-step and whole-solve parity
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("w", [S.TINY, SMALL_BF16, WIDE_BF16], ids=lambda w: w.name)
def test_velocity_and_solve_match_oracle(cuda_device, w):
    weights_cpu, weights, k, v, p, s = _setup(w)
    z0, eps = S.make_latents(w)
    eps = eps[0]
    taus = S.uniform_taus(w.n_steps)
    # one step with the velocity exposed
    z = eps.cuda().clone()
    vel = torch.empty_like(z)
    p.denoise_step(s, z, taus[0], taus[1], vel)
    torch.cuda.synchronize()
    ref_v = _oracle_velocity(w, weights_cpu, k, v, w.cache_units, eps, taus[0])
    e_v = rel_l2(vel.cpu().numpy(), ref_v)
    e_z1 = rel_l2(z.cpu().numpy(), O.euler_step(eps, ref_v, taus[0], taus[1]))
    # the whole solve
    z = eps.cuda().clone()
    p.fm_solve(s, z, taus)
    torch.cuda.synchronize()
    ck, cv = oracle_cache_layers(k, v, w.cache_units, w.unit_kv_tokens, w.cache_units)
    ref_z = O.denoise_solve(ocfg(w), eps, taus, weights_cpu, ck, cv,
                            w.cache_units * w.unit_kv_tokens, w.cache_units * w.unit_kv_tokens)
    e_z = rel_l2(z.cpu().numpy(), ref_z)
    print(f"{w.name}: velocity {e_v:.3e}  first step {e_z1:.3e}  solve {e_z:.3e}")
    assert e_v <= tol(w) and e_z1 <= tol(w) and e_z <= tol(w)
    p.close()


def test_velocity_with_random_norm_gains_matches_oracle(cuda_device):
    # the synthetic weights have unit RMSNorm gains; here every gain vector (both norms
    # of every layer and the final one) is drawn from U[0.5, 1.5], so each gain must be
    # applied at its own norm, including in the bf16 path where the norm is split
    # between the kernel that updates x and the next projection
    w = SMALL_BF16
    weights_cpu = S.make_weights(w)
    g = torch.Generator().manual_seed(31)
    def draw(t):
        return (0.5 + torch.rand(t.shape, generator=g)).to(t.dtype)
    weights_cpu["g_final"] = draw(weights_cpu["g_final"])
    for lay in weights_cpu["layers"]:
        lay["g_attn"] = draw(lay["g_attn"])
        lay["g_mlp"] = draw(lay["g_mlp"])
    weights = to_cuda(weights_cpu)
    k, v = S.make_kv_slices(w, w.cache_units)
    p = _performer(w, weights)
    s = p.open_session(w.cache_units)
    p.kvcache_append(s, k.cuda(), v.cuda())
    _, eps = S.make_latents(w)
    eps = eps[0]
    z = eps.cuda().clone()
    vel = torch.empty_like(z)
    p.denoise_step(s, z, 1.0, 0.75, vel)
    torch.cuda.synchronize()
    ref_v = _oracle_velocity(w, weights_cpu, k, v, w.cache_units, eps, 1.0)
    e_v = rel_l2(vel.cpu().numpy(), ref_v)
    print(f"random gains: velocity {e_v:.3e}")
    assert e_v <= BF16_TOL, e_v
    p.close()


def test_ring_wrapped_cache_velocity_matches_oracle(cuda_device):
    # 7 units into 5 slots: units 5, 6 overwrite slots 0, 1; positions keep counting
    w = SMALL_BF16
    weights_cpu, weights, k, v, p, s = _setup(w, n_units=7)
    info = p.session_info(s)
    assert info["units_appended"] == 7 and info["valid_tokens"] == 500 and info["p0"] == 700
    _, eps = S.make_latents(w)
    z = eps[0].cuda().clone()
    vel = torch.empty_like(z)
    p.denoise_step(s, z, 1.0, 0.75, vel)
    torch.cuda.synchronize()
    ref = _oracle_velocity(w, weights_cpu, k, v, 7, eps[0], 1.0)
    assert rel_l2(vel.cpu().numpy(), ref) <= BF16_TOL
    p.close()


def test_v01_full_denoise_step_matches_oracle(cuda_device):
    # 192x336 unit, 28 layers, full 64 x 512-token cache: one Euler step, all velocities
    w = S.V01
    weights_cpu, weights, k, v, p, s = _setup(w)
    _, eps = S.make_latents(w)
    z = eps[0].cuda().clone()
    vel = torch.empty_like(z)
    p.denoise_step(s, z, 1.0, 0.75, vel)
    torch.cuda.synchronize()
    ref = O.f_theta(ocfg(w), eps[0], 1.0, weights_cpu, list(k), list(v),
                    w.cache_units * w.unit_kv_tokens, w.cache_units * w.unit_kv_tokens)
    e = rel_l2(vel.cpu().numpy(), ref)
    print(f"v0.1 velocity rel L2 {e:.3e}")
    assert e <= BF16_TOL
    p.close()


def test_v02_width_full_cache_step_matches_oracle(cuda_device):
    # 640x368 unit at full width with the full 57,600-token cache; 2 layers so the
    # fp64 oracle stays in seconds (every layer runs the same kernels)
    w = S.V02.replace(n_layers=2)
    weights_cpu, weights, k, v, p, s = _setup(w)
    _, eps = S.make_latents(w)
    z = eps[0].cuda().clone()
    vel = torch.empty_like(z)
    p.denoise_step(s, z, 0.75, 0.5, vel)
    torch.cuda.synchronize()
    ref = O.f_theta(ocfg(w), eps[0], 0.75, weights_cpu, list(k), list(v), 57600, 57600)
    e = rel_l2(vel.cpu().numpy(), ref)
    print(f"v0.2-width velocity rel L2 {e:.3e}")
    assert e <= BF16_TOL
    p.close()


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

# a CTA takes 256 query rows as two 128-row tiles: 257 gives a second CTA with one
# row (its tile B empty), 300 a partial tile B, 513 a third CTA with one row
@pytest.mark.parametrize("n_q,n_kv", [(1, 1), (17, 5), (64, 64), (204, 704), (924, 5724),
                                      (257, 1), (300, 129), (513, 1000), (1030, 3000)])
def test_attention_bf16_matches_oracle(cuda_device, n_q, n_kv):
    from streaming_flow_matching_b200 import attention
    q, k, v = S.make_qkv(n_q, n_kv, 3, 128)
    o = attention(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    ref = O.attention(q, k, v)
    e = rel_l2(o.float().cpu().numpy(), ref)
    assert e <= BF16_TOL, e


@pytest.mark.parametrize("n_kv", S.ATTN_SWEEP_TOKENS)
def test_attention_sweep_sampled_rows(cuda_device, n_kv):
    # isolated attention at the sweep's cache lengths (+ the 924-token unit):
    # sampled query rows against the oracle, one row at a time
    from streaming_flow_matching_b200 import attention
    n_q, H = 924, 24
    q, k, v = S.make_qkv(n_q, n_kv + n_q, H, 128, device="cuda")
    o = attention(q, k, v)
    torch.cuda.synchronize()
    rows = [0, 1, 63, 64, 500, 895, 896, 923]
    ref = O.attention(q[rows].cpu(), k.cpu(), v.cpu())
    e = rel_l2(o[rows].float().cpu().numpy(), ref)
    assert e <= BF16_TOL, e


@pytest.mark.parametrize("n_q", [128, 640])
@pytest.mark.parametrize("n_kv", [512, 20000])
def test_attention_max_jump_in_some_rows_only(cuda_device, n_q, n_kv):
    # A few rows (one lane in each of several warps) meet a key aligned with their
    # query in a later key tile: their running max jumps by far more than 2^8 while
    # the rest of the warp's rows do not, so the online-softmax rescale of O is
    # needed by only some rows of a warp.
    from streaming_flow_matching_b200 import attention
    g = torch.Generator().manual_seed(21)
    H = 2
    q = torch.randn(n_q, H, 128, generator=g)
    k = 0.1 * torch.randn(n_kv, H, 128, generator=g)
    v = torch.randn(n_kv, H, 128, generator=g)
    rows = [3, 40, 77, 101] + ([300, 333, 600] if n_q > 128 else [])
    for i, r in enumerate(rows):
        k[300 + i] = 2.0 * q[r]
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    o = attention(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    e = rel_l2(o.float().cpu().numpy(), O.attention(q, k, v))
    assert e <= BF16_TOL, e


def test_attention_fp32_matches_oracle(cuda_device):
    from streaming_flow_matching_b200 import attention
    q, k, v = S.make_qkv(68, 452, 4, 64, dtype="fp32")
    o = attention(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert rel_l2(o.cpu().numpy(), O.attention(q, k, v)) <= FP32_TOL


# ---------------------------------------------------------------------------
# Euler update and the rectified-flow closed form
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n", [1, 7, 1 << 20, (1 << 24) + 3])
def test_euler_exact_velocity_returns_clean_latent(cuda_device, n):
    from streaming_flow_matching_b200 import euler_update
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    z0 = torch.randn(n, generator=g, device="cuda")
    eps = torch.randn(n, generator=g, device="cuda")
    vel = eps - z0
    z = eps.clone()
    taus = [1.0, 0.75, 0.5, 0.25, 0.0]
    for a, b in zip(taus[:-1], taus[1:]):
        euler_update(z, vel, b - a)
    torch.cuda.synchronize()
    assert rel_l2(z.cpu().numpy(), z0.cpu().numpy()) <= 1e-6
    z = eps.clone()
    euler_update(z, vel, -1.0)                       # one step 1 -> 0
    torch.cuda.synchronize()
    assert rel_l2(z.cpu().numpy(), z0.cpu().numpy()) <= 1e-6


@pytest.mark.parametrize("taus", [[1.0, 0.75, 0.5, 0.25, 0.0], [1.0, 0.9, 0.3, 0.05, 0.0], [1.0, 0.0]],
                         ids=["uniform4", "ragged4", "one-step"])
def test_solve_loop_with_exact_velocity_returns_clean_latent(cuda_device, taus):
    # the solve loop with f_theta replaced by the exact rectified-flow velocity
    # (z - z0) / tau ends at z0 for any schedule (closed form); evaluating the
    # velocity at a step's end point or stepping the wrong way would not
    from streaming_flow_matching_b200 import Performer
    w = S.TINY
    p = Performer.from_workload(w, to_cuda(S.make_weights(w)), pool_tokens=w.n_tokens + w.unit_kv_tokens)
    z0, eps = S.make_latents(w, device="cuda")
    z = eps[0].clone()
    p.fm_solve_exact_velocity(z0[0], z, taus)
    torch.cuda.synchronize()
    assert rel_l2(z.cpu().numpy(), z0[0].cpu().numpy()) <= 1e-6
    p.close()
