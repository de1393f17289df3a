"""Oracle parity at the shapes the benchmark and the results table time, through the
C ABI: the 640x368 unit at full depth (28 layers, full 57,600-token cache, the whole
4-step solve), eight ragged sessions batched at the 640x368 width, and a guided step
at that width.  Tolerance: relative L2 <= 2e-2 on bf16 velocities and latents.
"""
import numpy as np
import pytest
import torch

import sfm_synth as S
from oracle import sfm_oracle as O
from tests._gpu_util import BF16_TOL, ocfg, rel_l2, to_cuda
from tests.golden import make_v02_golden as G

pytestmark = pytest.mark.gpu


def _performer(w, weights, caps):
    from streaming_flow_matching_b200 import Performer
    pool = sum(c * w.unit_kv_tokens + w.n_tokens for c in caps)
    return Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=len(caps))


def test_v02_full_depth_solve_matches_stored_oracle(cuda_device):
    # 28 layers, d = 3072, 24 heads, F = 12288, 924 tokens over 57,600 cached tokens:
    # the first step's velocity and latent and the whole 4-step solve against the fp64
    # oracle's values, stored by tests/golden/make_v02_golden.py (oracle only; tens of
    # minutes on a CPU).  The inputs are redrawn here and must match the fingerprint
    # the stored values were computed on.
    gold = np.load(G.OUT)
    w = S.V02
    weights_cpu = S.make_weights(w)
    _, eps = S.make_latents(w)
    eps = eps[0]
    fp = G.fingerprint_head(weights_cpu, eps)
    shape = (w.n_layers, w.cache_units * w.unit_kv_tokens, w.n_heads, w.head_dim)
    k = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    v = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    for layer in range(w.n_layers):
        kl, vl = S.make_kv_layer(w, w.cache_units, layer)
        fp += G.fingerprint_layer(kl, vl)
        k[layer].copy_(kl)
        v[layer].copy_(vl)
    assert np.array_equal(np.array(fp), gold["fingerprint"]), "seeded inputs differ from the stored run"
    p = _performer(w, to_cuda(weights_cpu), [w.cache_units])
    s = p.open_session(w.cache_units)
    p.kvcache_append(s, k, v)
    del k, v
    taus = [float(t) for t in gold["taus"]]
    z = eps.cuda().clone()
    vel = torch.empty_like(z)
    p.denoise_step(s, z, taus[0], taus[1], vel)
    torch.cuda.synchronize()
    e_v = rel_l2(vel.cpu().numpy(), gold["v_step0"])
    e_z1 = rel_l2(z.cpu().numpy(), gold["z_step1"])
    z = eps.cuda().clone()
    p.fm_solve(s, z, taus)
    torch.cuda.synchronize()
    e_z = rel_l2(z.cpu().numpy(), gold["z_solve"])
    print(f"v0.2 28 layers: velocity {e_v:.3e}  first step {e_z1:.3e}  4-step solve {e_z:.3e}")
    assert p.check_device_error() == 0
    assert e_v <= BF16_TOL and e_z1 <= BF16_TOL and e_z <= BF16_TOL
    p.close()


def test_eight_ragged_sessions_at_640x368_width_match_oracle(cuda_device):
    # the 8-session throughput configuration at full width (2 layers so the oracle
    # stays in seconds): caches drawn in [8K, 64K] tokens, one batched Euler step;
    # at M = 8 x 924 rows the residual projections (O, MLP-down) run on CTA pairs
    # with the next RMSNorm's numerator and sums of squares fused into their epilogue
    w = S.V02X8.replace(n_layers=2)
    caps = S.session_cache_units(unit_tokens=w.unit_kv_tokens)
    weights_cpu = S.make_weights(w)
    p = _performer(w, to_cuda(weights_cpu), caps)
    plan = p.plan()
    assert plan["pair"][1] == 1 and plan["pair"][3] == 1 and plan["fused_norm"] == 1, plan
    check = sorted({int(np.argmax(caps)), int(np.argmin(caps)), 3})
    sessions, kept = [], {}
    for i, cap in enumerate(caps):
        s = p.open_session(cap)
        k, v = S.make_kv_slices(w, cap, seed=S.SEED_CACHE + 10 * i)
        p.kvcache_append(s, k.cuda(), v.cuda())
        sessions.append(s)
        if i in check:
            kept[i] = (k, v)
    _, eps = S.make_latents(w, n_sessions=len(caps))
    zs = [eps[i].cuda().clone() for i in range(len(caps))]
    taus = [1.0, 0.75]
    p.fm_solve_batched(sessions, zs, taus)
    torch.cuda.synchronize()
    assert p.check_device_error() == 0
    for i in check:
        k, v = kept[i]
        valid = caps[i] * w.unit_kv_tokens
        ref_v = O.f_theta(ocfg(w), eps[i], taus[0], weights_cpu, list(k), list(v), valid, valid)
        got_z = zs[i].cpu().double().numpy()
        e_z = rel_l2(got_z, O.euler_step(eps[i], ref_v, taus[0], taus[1]))
        # the step's velocity, recovered from the latent it moved (fp32 z: ~1e-7 error)
        got_v = (got_z - eps[i].double().numpy()) / (taus[1] - taus[0])
        e_v = rel_l2(got_v, ref_v)
        print(f"session {i}: {valid} cached tokens: velocity {e_v:.3e}  latent {e_z:.3e}")
        assert e_v <= BF16_TOL and e_z <= BF16_TOL
    p.close()


def test_guided_step_at_640x368_width_matches_oracle(cuda_device):
    # classifier-free guidance at full width: conditional context = the full
    # 57,600-token cache, unconditional = an empty session; 2 layers
    w = S.V02.replace(n_layers=2)
    weights_cpu = S.make_weights(w)
    p = _performer(w, to_cuda(weights_cpu), [w.cache_units, 1])
    s = p.open_session(w.cache_units)
    u = p.open_session(1)
    k, v = S.make_kv_slices(w, w.cache_units)
    p.kvcache_append(s, k.cuda(), v.cuda())
    _, eps = S.make_latents(w)
    eps = eps[0]
    scale = 3.5
    z = eps.cuda().clone()
    vel = torch.empty_like(z)
    p.fm_solve_guided_batched([s], [u], [z], [1.0, 0.75], scale, v_outs=[vel])
    torch.cuda.synchronize()
    cfg = ocfg(w)
    valid = w.cache_units * w.unit_kv_tokens
    v_c = O.f_theta(cfg, eps, 1.0, weights_cpu, list(k), list(v), valid, valid)
    empty = [np.zeros((0, w.n_heads, w.head_dim))] * w.n_layers
    v_u = O.f_theta(cfg, eps, 1.0, weights_cpu, empty, empty, 0, 0)
    ref_v = O.guided_velocity(v_c, v_u, scale)
    e_v = rel_l2(vel.cpu().numpy(), ref_v)
    e_z = rel_l2(z.cpu().numpy(), O.euler_step(eps, ref_v, 1.0, 0.75))
    print(f"guided at 640x368 width: velocity {e_v:.3e}  latent {e_z:.3e}")
    assert p.check_device_error() == 0
    assert e_v <= BF16_TOL and e_z <= BF16_TOL
    p.close()
