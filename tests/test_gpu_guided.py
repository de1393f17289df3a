"""Classifier-free-guided solves through the C ABI against the oracle's guided
solve: v = v_u + s (v_c - v_u) at every Euler step, both evaluations at the
same z.  The unconditional context is an empty session (the unit attends to
itself alone) or a session holding a different context; guided batches of
several pairs; argument errors.  Tolerances as for plain solves: relative L2
<= 1e-5 in the fp32 mode and <= 2e-2 in bf16."""
import numpy as np
import pytest
import torch

import sfm_synth as S
from oracle import sfm_oracle as O
from tests._gpu_util import SMALL_BF16, ocfg, oracle_cache_layers, rel_l2, to_cuda, tol

pytestmark = pytest.mark.gpu

SEED_NULL = 77          # K/V of the "null prompt" unconditional context


def _performer(w, weights, caps):
    from streaming_flow_matching_b200 import Performer
    pool = sum(c * w.unit_kv_tokens + w.n_tokens for c in caps)
    return Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=len(caps))


def _context(w, p, s, n_units, seed):
    """Appends n_units seeded units to session s; returns the oracle's view of it."""
    if n_units == 0:
        empty = [np.zeros((0, w.n_heads, w.head_dim))] * w.n_layers
        return (empty, empty, 0, 0)
    k, v = S.make_kv_slices(w, n_units, seed=seed)
    p.kvcache_append(s, k.cuda(), v.cuda())
    ck, cv = oracle_cache_layers(k, v, n_units, w.unit_kv_tokens, n_units)
    T = n_units * w.unit_kv_tokens
    return (ck, cv, T, T)


@pytest.mark.parametrize("w", [S.TINY, SMALL_BF16], ids=lambda w: w.name)
@pytest.mark.parametrize("null_units", [0, 1], ids=["empty-null", "null-prompt"])
def test_guided_step_and_solve_match_oracle(cuda_device, w, null_units):
    weights_cpu = S.make_weights(w)
    p = _performer(w, to_cuda(weights_cpu), [w.cache_units, max(null_units, 1)])
    s = p.open_session(w.cache_units)
    u = p.open_session(max(null_units, 1))
    cond = _context(w, p, s, w.cache_units, S.SEED_CACHE)
    uncond = _context(w, p, u, null_units, SEED_NULL)
    _, eps = S.make_latents(w)
    eps = eps[0]
    scale = 3.5
    taus = S.uniform_taus(w.n_steps)
    cfg = ocfg(w)
    # one step, guided velocity exposed
    z = eps.cuda().clone()
    vel = torch.empty_like(z)
    p.fm_solve_guided_batched([s], [u], [z], taus[:2], scale, v_outs=[vel])
    torch.cuda.synchronize()
    v_c = O.f_theta(cfg, eps, taus[0], weights_cpu, *cond)
    v_u = O.f_theta(cfg, eps, taus[0], weights_cpu, *uncond)
    ref_v = O.guided_velocity(v_c, v_u, scale)
    e_v = rel_l2(vel.cpu().numpy(), ref_v)
    e_z1 = rel_l2(z.cpu().numpy(), O.euler_step(eps, ref_v, taus[0], taus[1]))
    # the whole guided solve
    z = eps.cuda().clone()
    p.fm_solve_guided(s, u, z, taus, scale)
    torch.cuda.synchronize()
    ref_z = O.denoise_solve_cfg(cfg, eps, taus, weights_cpu, cond, uncond, scale)
    e_z = rel_l2(z.cpu().numpy(), ref_z)
    print(f"{w.name} null units {null_units}: guided velocity {e_v:.3e}  first step {e_z1:.3e}  "
          f"solve {e_z:.3e}")
    assert e_v <= tol(w) and e_z1 <= tol(w) and e_z <= tol(w)
    # neither cache changed: the guided solve appends nothing
    assert p.session_info(s)["units_appended"] == w.cache_units
    assert p.session_info(u)["units_appended"] == null_units
    assert p.check_device_error() == 0
    p.close()


def test_guided_batch_of_pairs_matches_oracle(cuda_device):
    # three pairs with different cache lengths and contexts in one batch of six
    w = S.TINY
    weights_cpu = S.make_weights(w)
    caps = [w.cache_units, 2, 3, 1, 4, 1]
    p = _performer(w, to_cuda(weights_cpu), caps)
    ids = [p.open_session(c) for c in caps]
    fills = [w.cache_units, 2, 3, 0, 1, 0]
    ctx = [_context(w, p, ids[i], fills[i], S.SEED_CACHE + 10 * i) for i in range(6)]
    _, eps = S.make_latents(w, n_sessions=3)
    taus = S.uniform_taus(w.n_steps)
    scale = 2.0
    zs = [eps[i].cuda().clone() for i in range(3)]
    p.fm_solve_guided_batched(ids[0::2], ids[1::2], zs, taus, scale)
    torch.cuda.synchronize()
    for i in range(3):
        ref = O.denoise_solve_cfg(ocfg(w), eps[i], taus, weights_cpu, ctx[2 * i], ctx[2 * i + 1],
                                  scale)
        e = rel_l2(zs[i].cpu().numpy(), ref)
        assert e <= tol(w), f"pair {i}: {e:.3e}"
    p.close()


def test_guided_scale_zero_and_one_reduce_to_plain_solves(cuda_device):
    # s = 1 follows the conditional velocity, s = 0 the unconditional one; the
    # guided batch rounds differently from a plain one only at the fp32 level
    w = S.TINY
    weights = to_cuda(S.make_weights(w))
    p = _performer(w, weights, [w.cache_units, 2])
    s = p.open_session(w.cache_units)
    u = p.open_session(2)
    k, v = S.make_kv_slices(w, w.cache_units)
    p.kvcache_append(s, k.cuda(), v.cuda())
    k2, v2 = S.make_kv_slices(w, 2, seed=SEED_NULL)
    p.kvcache_append(u, k2.cuda(), v2.cuda())
    _, eps = S.make_latents(w)
    eps = eps[0].cuda()
    taus = S.uniform_taus(w.n_steps)
    out = {}
    for name, call in (("cond", lambda z: p.fm_solve(s, z, taus)),
                       ("uncond", lambda z: p.fm_solve(u, z, taus)),
                       ("g1", lambda z: p.fm_solve_guided(s, u, z, taus, 1.0)),
                       ("g0", lambda z: p.fm_solve_guided(s, u, z, taus, 0.0))):
        z = eps.clone()
        call(z)
        torch.cuda.synchronize()
        out[name] = z.cpu().numpy()
    assert rel_l2(out["cond"], out["uncond"]) > 1e-3
    assert rel_l2(out["g1"], out["cond"]) <= 1e-6
    assert rel_l2(out["g0"], out["uncond"]) <= 1e-6
    p.close()


def test_guided_argument_errors(cuda_device):
    from streaming_flow_matching_b200 import _lib as L
    w = S.TINY
    weights = to_cuda(S.make_weights(w))
    p = _performer(w, weights, [2, 1])
    s = p.open_session(2)
    u = p.open_session(1)
    z = torch.zeros(w.n_tokens, w.c_lat, device="cuda")
    taus = S.uniform_taus(2)
    with pytest.raises(L.SfmError) as e:
        p.fm_solve_guided(s, s, z, taus, 2.0)           # same session twice
    assert e.value.status == L.SFM_EINVAL
    with pytest.raises(L.SfmError) as e:
        p.fm_solve_guided(s, u, z, taus, float("nan"))
    assert e.value.status == L.SFM_EINVAL
    with pytest.raises(L.SfmError) as e:
        p.fm_solve_guided(s, 5, z, taus, 2.0)           # no such session
    assert e.value.status == L.SFM_ESESSION
    with pytest.raises(L.SfmError) as e:                # 4 evaluations > max_sessions = 2
        p.fm_solve_guided_batched([s, u], [u, s], [z, z.clone()], taus, 2.0)
    assert e.value.status == L.SFM_ECAPACITY
    p.close()
    # two pairs sharing one latent buffer: both Euler updates would write it
    p4 = _performer(w, weights, [2, 1, 2, 1])
    ids = [p4.open_session(c) for c in (2, 1, 2, 1)]
    with pytest.raises(L.SfmError) as e:
        p4.fm_solve_guided_batched(ids[0::2], ids[1::2], [z, z], taus, 2.0)
    assert e.value.status == L.SFM_EINVAL
    z2 = z.clone()
    with pytest.raises(L.SfmError) as e:                # a velocity output that is a latent
        p4.fm_solve_guided_batched(ids[0::2], ids[1::2], [z, z2], taus, 2.0, v_outs=[z2, None])
    assert e.value.status == L.SFM_EINVAL
    with pytest.raises(L.SfmError) as e:
        p4.denoise_step(ids[0], z, 1.0, 0.5, z)
    assert e.value.status == L.SFM_EINVAL
    p4.close()
    # one session per handle: no room for the unconditional evaluation
    p1 = _performer(w, weights, [2])
    s1 = p1.open_session(2)
    with pytest.raises(L.SfmError) as e:
        p1.fm_solve_guided(s1, s1, z, taus, 2.0)
    assert e.value.status == L.SFM_ECAPACITY
    p1.close()
