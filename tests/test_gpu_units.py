"""Several units in one pass of f_theta under the general block-causal mask
(sfm_velocity_units) against the oracle: with no cache it is the masked
full-sequence form, after a cache the oracle's multi-unit pass; one unit equals
the denoise step's velocity bit for bit; committing appends the units' own K/V,
after which the next unit's step sees them as cache."""
import ctypes as C

import numpy as np
import pytest
import torch

import sfm_synth as S
from oracle import sfm_oracle as O
from streaming_flow_matching_b200 import SfmError, _lib as L
from tests._gpu_util import SMALL_BF16, ocfg, oracle_cache_layers, rel_l2, to_cuda, tol

pytestmark = pytest.mark.gpu


def _performer(w, weights, cache_units, max_sessions):
    from streaming_flow_matching_b200 import Performer
    pool = cache_units * w.unit_kv_tokens + w.n_tokens
    return Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=max_sessions)


def _latents(w, n, seed=60):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(w.n_tokens, w.c_lat, generator=g) for _ in range(n)]


@pytest.mark.parametrize("w", [S.TINY, SMALL_BF16], ids=lambda w: w.name)
@pytest.mark.parametrize("cached", [0, 2], ids=["no-cache", "after-cache"])
def test_units_pass_matches_oracle(cuda_device, w, cached):
    n_units, cu = 3, 10          # room for the cache and the pass's 3 N rows
    weights_cpu = S.make_weights(w)
    p = _performer(w, to_cuda(weights_cpu), cu, n_units)
    s = p.open_session(cu)
    ck = cv = [np.zeros((0, w.n_heads, w.head_dim))] * w.n_layers
    if cached:
        k, v = S.make_kv_slices(w, cached)
        p.kvcache_append(s, k.cuda(), v.cuda())
        ck, cv = oracle_cache_layers(k, v, cached, w.unit_kv_tokens, cu)
    zs = _latents(w, n_units)
    taus = [0.0, 0.5, 1.0]
    vel = p.velocity_units(s, [z.cuda() for z in zs], taus)
    torch.cuda.synchronize()
    valid = cached * w.unit_kv_tokens
    ref = O.f_theta_units(ocfg(w), zs, taus, weights_cpu, ck, cv, valid, valid)
    if not cached:
        seq = O.f_theta_sequence(ocfg(w), zs, taus, weights_cpu)
        for a, b in zip(ref, seq):
            np.testing.assert_allclose(a, b, atol=1e-10)
    for u in range(n_units):
        e = rel_l2(vel[u].cpu().numpy(), ref[u])
        print(f"{w.name} cached {cached} unit {u}: rel L2 {e:.3e}")
        assert e <= tol(w), (u, e)
    # nothing was committed
    assert p.session_info(s)["units_appended"] == cached
    assert p.check_device_error() == 0
    p.close()


def test_units_pass_at_640x368_width_over_a_cache(cuda_device):
    # four 924-token units after a 12-unit (14,400-token) cache, 24 heads x 128,
    # d = 3072, 2 layers: the block-causal attention over 18,096 keys at M = 3696
    w = S.V02.replace(n_layers=2, cache_units=48)
    n_units, cached = 4, 12
    weights_cpu = S.make_weights(w)
    p = _performer(w, to_cuda(weights_cpu), w.cache_units, n_units)
    s = p.open_session(w.cache_units)
    k, v = S.make_kv_slices(w, cached)
    p.kvcache_append(s, k.cuda(), v.cuda())
    zs = _latents(w, n_units, seed=61)
    taus = [0.0, 0.0, 0.0, 0.75]
    vel = p.velocity_units(s, [z.cuda() for z in zs], taus)
    torch.cuda.synchronize()
    valid = cached * w.unit_kv_tokens
    ref = O.f_theta_units(ocfg(w), zs, taus, weights_cpu, list(k), list(v), valid, valid)
    for u in range(n_units):
        e = rel_l2(vel[u].cpu().numpy(), ref[u])
        print(f"640x368 width unit {u}: rel L2 {e:.3e}")
        assert e <= tol(w)
    p.close()


@pytest.mark.parametrize("w", [S.TINY, SMALL_BF16], ids=lambda w: w.name)
def test_one_unit_pass_equals_the_denoise_step_velocity(cuda_device, w):
    weights_cpu = S.make_weights(w)
    p = _performer(w, to_cuda(weights_cpu), w.cache_units, 1)
    s = p.open_session(w.cache_units)
    k, v = S.make_kv_slices(w, 2)
    p.kvcache_append(s, k.cuda(), v.cuda())
    z = _latents(w, 1)[0].cuda()
    vel = p.velocity_units(s, [z], [0.75])[0]
    z2 = z.clone()
    vel2 = torch.empty_like(z)
    p.denoise_step(s, z2, 0.75, 0.5, vel2)
    torch.cuda.synchronize()
    assert torch.equal(vel, vel2)
    assert torch.equal(z, _latents(w, 1)[0].cuda())      # the pass only reads z
    p.close()


@pytest.mark.parametrize("w", [S.TINY.replace(unit_kv_tokens=68),
                               SMALL_BF16.replace(unit_kv_tokens=204)], ids=lambda w: w.name)
def test_commit_appends_the_units_own_kv(cuda_device, w):
    # a cache unit of N tokens: two clean units (tau = 0) committed, then the next
    # unit's step sees their K/V as its cache (positions continue)
    weights_cpu = S.make_weights(w)
    p = _performer(w, to_cuda(weights_cpu), 4, 2)
    s = p.open_session(4)
    zs = _latents(w, 3, seed=62)
    vel = p.velocity_units(s, [z.cuda() for z in zs[:2]], [0.0, 0.0], commit=True)
    torch.cuda.synchronize()
    info = p.session_info(s)
    assert info["units_appended"] == 2 and info["valid_tokens"] == 2 * w.n_tokens
    assert info["p0"] == 2 * w.n_tokens
    empty = [np.zeros((0, w.n_heads, w.head_dim))] * w.n_layers
    ref3, kv = O.f_theta_units(ocfg(w), zs, [0.0, 0.0, 0.6], weights_cpu, empty, empty, 0, 0,
                               return_kv=True)
    for u in range(2):
        assert rel_l2(vel[u].cpu().numpy(), ref3[u]) <= tol(w)
    n = w.n_tokens
    for layer in range(w.n_layers):
        kc, vc = p.kvcache_read(s, layer, 0, 2 * n)
        torch.cuda.synchronize()
        assert rel_l2(kc.float().cpu().numpy(), kv[layer][0][:2 * n]) <= tol(w)
        assert rel_l2(vc.float().cpu().numpy(), kv[layer][1][:2 * n]) <= tol(w)
    # the third unit's velocity through the plain step over the committed cache
    z3 = zs[2].cuda().clone()
    v3 = torch.empty_like(z3)
    p.denoise_step(s, z3, 0.6, 0.3, v3)
    torch.cuda.synchronize()
    e = rel_l2(v3.cpu().numpy(), ref3[2])
    print(f"{w.name}: unit after two committed units rel L2 {e:.3e}")
    assert e <= tol(w)
    p.close()


def test_units_argument_errors(cuda_device):
    w = SMALL_BF16
    p = _performer(w, to_cuda(S.make_weights(w)), w.cache_units, 2)
    s = p.open_session(w.cache_units)
    zs = [z.cuda() for z in _latents(w, 3)]
    st = C.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call(zz, vv, taus, commit=0, n=None, sess=s):
        n = len(zz) if n is None else n
        zp = (C.c_void_p * max(1, len(zz)))(*[t.data_ptr() for t in zz])
        vp = (C.c_void_p * max(1, len(vv)))(*[t.data_ptr() for t in vv])
        tp = (C.c_float * max(1, len(taus)))(*taus)
        return L.lib.sfm_velocity_units(p._h, sess, n, zp, tp, vp, commit, st)

    outs = [torch.empty_like(z) for z in zs]
    assert call(zs, outs, [0.0] * 3) == L.SFM_ECAPACITY            # more units than max_sessions
    assert call(zs[:2], [outs[0], outs[0]], [0.0] * 2) == L.SFM_EINVAL   # one buffer twice
    assert call(zs[:2], [outs[0], zs[1]], [0.0] * 2) == L.SFM_EINVAL     # v_out is a latent
    assert call(zs[:1], outs[:1], [float("nan")]) == L.SFM_EINVAL
    assert call(zs[:1], outs[:1], [0.0], commit=1) == L.SFM_EUNSUPPORTED  # T_u != N
    assert call(zs[:1], outs[:1], [0.0], commit=2) == L.SFM_EINVAL
    assert call(zs[:1], outs[:1], [0.0], sess=5) == L.SFM_ESESSION
    assert call([], [], [], n=0) == L.SFM_EINVAL
    # a full 5-unit cache leaves room for one unit's rows only
    k, v = S.make_kv_slices(w, w.cache_units)
    p.kvcache_append(s, k.cuda(), v.cuda())
    assert call(zs[:2], outs[:2], [0.0] * 2) == L.SFM_ECAPACITY
    assert call(zs[:1], outs[:1], [0.0]) == L.SFM_OK
    torch.cuda.synchronize()
    p.close()
