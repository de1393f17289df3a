"""Pins of the fp64 oracle against what the pages and mathematics fix.

Each test ties one oracle step to something other than the oracle itself: a
closed form, an invariant the method must satisfy, a library routine, or a
scalar-loop brute force at toy size.  A plausible slip in the oracle (dropped
term, wrong sign, swapped index, transposed operand) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

from oracle import sfm_oracle as O
from tests import _bruteforce as BF

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny_cfg(**kw):
    base = dict(n_layers=2, d_model=8, n_heads=2, head_dim=4, d_mlp=16, c_lat=3,
                n_video=3, n_audio=2, unit_kv_tokens=5)
    base.update(kw)
    return O.Config(**base)


def tiny_weights(cfg, rng, std=0.3):
    """Random tiny weights; non-unit gains so a dropped gain shows up."""
    n = lambda *s: rng.standard_normal(s) * std
    w = {"w_in": n(cfg.d_model, cfg.c_lat), "e_mod": n(2, cfg.d_model),
         "g_final": 1.0 + 0.1 * rng.standard_normal(cfg.d_model),
         "w_out": n(cfg.c_lat, cfg.d_model), "layers": []}
    for _ in range(cfg.n_layers):
        w["layers"].append({
            "g_attn": 1.0 + 0.1 * rng.standard_normal(cfg.d_model),
            "w_qkv": n(3 * cfg.hd, cfg.d_model), "w_o": n(cfg.d_model, cfg.hd),
            "g_mlp": 1.0 + 0.1 * rng.standard_normal(cfg.d_model),
            "w_1": n(cfg.d_mlp, cfg.d_model), "w_2": n(cfg.d_model, cfg.d_mlp)})
    return w


# --------------------------------------------------------------------------
# rectified-flow path and the Euler solve
# --------------------------------------------------------------------------

def test_rf_path_endpoints_and_velocity():
    rng = np.random.default_rng(0)
    z0, eps = rng.standard_normal((5, 3)), rng.standard_normal((5, 3))
    assert np.array_equal(O.rf_path(z0, eps, 0.0), z0)          # tau = 0: clean latent
    assert np.array_equal(O.rf_path(z0, eps, 1.0), eps)         # tau = 1: pure noise
    h = 1e-6
    fd = (O.rf_path(z0, eps, 0.4 + h) - O.rf_path(z0, eps, 0.4 - h)) / (2 * h)
    np.testing.assert_allclose(fd, O.rf_velocity(z0, eps), atol=1e-8)


def test_single_euler_step_from_noise_returns_clean_latent():
    rng = np.random.default_rng(1)
    z0, eps = rng.standard_normal((7, 4)), rng.standard_normal((7, 4))
    v = O.rf_velocity(z0, eps)
    z = O.fm_solve(eps, [1.0, 0.0], lambda z, t: v)
    np.testing.assert_allclose(z, z0, rtol=0, atol=1e-15)


@pytest.mark.parametrize("n_steps", [1, 2, 4, 7, 32])
def test_any_schedule_with_exact_velocity_returns_clean_latent(n_steps):
    rng = np.random.default_rng(n_steps)
    z0, eps = rng.standard_normal((9, 16)), rng.standard_normal((9, 16))
    inner = np.sort(rng.uniform(0, 1, n_steps - 1))[::-1]
    taus = [1.0] + list(inner) + [0.0]
    v = O.rf_velocity(z0, eps)
    np.testing.assert_allclose(O.fm_solve(eps, taus, lambda z, t: v), z0, atol=1e-13)
    np.testing.assert_allclose(O.fm_solve(eps, O.uniform_taus(n_steps), lambda z, t: v),
                               z0, atol=1e-13)


def test_state_dependent_exact_velocity_stays_on_the_path():
    # On the linear path, (z_tau - z0) / tau is the velocity at (z_tau, tau); an Euler
    # step that evaluates it at the step's start time lands exactly on the path again.
    rng = np.random.default_rng(2)
    z0, eps = rng.standard_normal((6, 4)), rng.standard_normal((6, 4))
    taus = [1.0, 0.8, 0.55, 0.3, 0.1, 0.0]
    z = eps
    for i in range(len(taus) - 1):
        z = O.euler_step(z, (z - z0) / taus[i], taus[i], taus[i + 1])
        np.testing.assert_allclose(z, O.rf_path(z0, eps, taus[i + 1]), atol=1e-13)
    np.testing.assert_allclose(O.fm_solve(eps, taus, lambda zz, t: (zz - z0) / t), z0, atol=1e-13)


def test_uniform_schedule():
    assert O.uniform_taus(4) == [1.0, 0.75, 0.5, 0.25, 0.0]
    assert O.uniform_taus(2) == [1.0, 0.5, 0.0]


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def test_attention_brute_force_tiny():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((5, 2, 4))
    k = rng.standard_normal((9, 2, 4))
    v = rng.standard_normal((9, 2, 4))
    out = O.attention(q, k, v)
    for i in range(5):
        for h in range(2):
            ref = BF.attend(list(q[i, h]), [list(k[j, h]) for j in range(9)],
                            [list(v[j, h]) for j in range(9)])
            np.testing.assert_allclose(out[i, h], ref, atol=1e-14)


def test_attention_matches_library_softmax():
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal(s) for s in ((6, 3, 8), (20, 3, 8), (20, 3, 8)))
    out = O.attention(q, k, v)
    for h in range(3):
        p = scipy.special.softmax(q[:, h] @ k[:, h].T / math.sqrt(8), axis=1)
        np.testing.assert_allclose(out[:, h], p @ v[:, h], atol=1e-14)


def test_attention_special_cases():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((4, 2, 8))
    v = rng.standard_normal((6, 2, 8))
    # a single key: the output is that key's value
    np.testing.assert_allclose(O.attention(q, rng.standard_normal((1, 2, 8)), v[:1]),
                               np.broadcast_to(v[:1], (4, 2, 8)), atol=1e-15)
    # identical keys or all-zero keys: the plain mean of the values
    same = np.broadcast_to(rng.standard_normal((1, 2, 8)), (6, 2, 8))
    mean = np.broadcast_to(v.mean(axis=0, keepdims=True), (4, 2, 8))
    np.testing.assert_allclose(O.attention(q, same, v), mean, atol=1e-14)
    np.testing.assert_allclose(O.attention(q, np.zeros((6, 2, 8)), v), mean, atol=1e-14)


def test_attention_two_key_closed_form_and_scale():
    # D = 4, one query e0, keys 2 e0 and 0: logits 2/sqrt(4) = 1 and 0, so
    # p0 = e / (1 + e) -- pins the 1/sqrt(D) scale and the softmax direction.
    q = np.zeros((1, 1, 4)); q[0, 0, 0] = 1.0
    k = np.zeros((2, 1, 4)); k[0, 0, 0] = 2.0
    v = np.zeros((2, 1, 4)); v[0, 0, 1] = 1.0; v[1, 0, 2] = 1.0
    p0 = math.e / (1.0 + math.e)
    np.testing.assert_allclose(O.attention(q, k, v)[0, 0], [0, p0, 1 - p0, 0], atol=1e-15)


def test_block_causal_mask():
    vis = O.block_causal_visible([0, 0, 1, 1], [0, 0, 1, 1])
    assert vis.tolist() == [[True, True, False, False], [True, True, False, False],
                            [True, True, True, True], [True, True, True, True]]
    rng = np.random.default_rng(6)
    q = rng.standard_normal((4, 1, 4)); k = rng.standard_normal((4, 1, 4)); v = rng.standard_normal((4, 1, 4))
    out = O.attention(q, k, v, vis)
    np.testing.assert_allclose(out[:2], O.attention(q[:2], k[:2], v[:2]), atol=1e-15)


def test_masked_attention_with_prefix_brute_force():
    # the form a multi-unit pass uses: prefix keys in unit -1 (visible to every query),
    # then the queries' own keys in units of uneven length; each row against the
    # scalar-loop attention over exactly the keys it may see
    q_units = [0, 0, 0, 1, 1, 2]
    k_units = [-1, -1] + q_units
    vis = O.block_causal_visible(q_units, k_units)
    rng = np.random.default_rng(7)
    q = rng.standard_normal((6, 2, 4))
    k = rng.standard_normal((8, 2, 4))
    v = rng.standard_normal((8, 2, 4))
    out = O.attention(q, k, v, vis)
    for i in range(6):
        seen = [j for j in range(8) if k_units[j] <= q_units[i]]
        assert len(seen) == 2 + sum(1 for u in q_units if u <= q_units[i])
        for h in range(2):
            ref = BF.attend(list(q[i, h]), [list(k[j, h]) for j in seen], [list(v[j, h]) for j in seen])
            np.testing.assert_allclose(out[i, h], ref, atol=1e-14)


# --------------------------------------------------------------------------
# RMSNorm, RoPE, GELU, tau embedding, linear
# --------------------------------------------------------------------------

def test_rmsnorm_closed_forms():
    g = np.array([1.0, 2.0, -3.0, 0.5])
    c = np.full((1, 4), -2.5)
    np.testing.assert_allclose(O.rmsnorm(c, g, 0.0), -g[None, :], atol=1e-15)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, 16))
    y = O.rmsnorm(x, np.ones(16), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=1), 1.0, atol=1e-14)
    np.testing.assert_allclose(O.rmsnorm(7.0 * x, np.ones(16), 0.0), y, atol=1e-14)
    # eps enters under the root: a zero row stays zero, a row of 1e-3 gives 1e-3/sqrt(1e-6+eps)
    np.testing.assert_allclose(O.rmsnorm(np.full((1, 4), 1e-3), np.ones(4), 1e-6),
                               np.full((1, 4), 1e-3 / math.sqrt(2e-6)), rtol=1e-14)


def test_rope_closed_forms():
    rng = np.random.default_rng(8)
    # D = 2: one pair rotated by p * theta^0 = p radians, counter-clockwise
    x = np.array([[[1.0, 0.0]]])
    np.testing.assert_allclose(O.rope(x, [1.0], 10000.0)[0, 0], [math.cos(1), math.sin(1)], atol=1e-15)
    x = np.array([[[0.0, 1.0]]])
    np.testing.assert_allclose(O.rope(x, [1.0], 10000.0)[0, 0], [-math.sin(1), math.cos(1)], atol=1e-15)
    # D = 4, theta = 1e4: second pair (x1, x3) turns by p * 1e4^(-1/2) = p / 100
    x = np.array([[[0.0, 1.0, 0.0, 0.0]]])
    np.testing.assert_allclose(O.rope(x, [50.0], 10000.0)[0, 0],
                               [0, math.cos(0.5), 0, math.sin(0.5)], atol=1e-15)
    # position 0 is the identity; pair norms are preserved
    x = rng.standard_normal((3, 2, 8))
    np.testing.assert_allclose(O.rope(x, [0, 0, 0], 1e4), x, atol=0)
    y = O.rope(x, [5, 17, 1000], 1e4)
    np.testing.assert_allclose(x[..., :4] ** 2 + x[..., 4:] ** 2, y[..., :4] ** 2 + y[..., 4:] ** 2, atol=1e-13)
    # q . k depends only on the position difference
    q, k = rng.standard_normal((1, 1, 8)), rng.standard_normal((1, 1, 8))
    d1 = np.sum(O.rope(q, [12], 1e4) * O.rope(k, [5], 1e4))
    d2 = np.sum(O.rope(q, [1012], 1e4) * O.rope(k, [1005], 1e4))
    assert abs(d1 - d2) < 1e-12


def test_gelu_tanh_pins():
    x = np.linspace(-6, 6, 241)
    exact = 0.5 * x * (1.0 + scipy.special.erf(x / math.sqrt(2.0)))
    assert np.max(np.abs(O.gelu_tanh(x) - exact)) < 1e-3
    # odd-part identity GELU(x) - GELU(-x) = x holds for the tanh form too
    np.testing.assert_allclose(O.gelu_tanh(x) - O.gelu_tanh(-x), x, atol=1e-14)
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert abs(O.gelu_tanh(np.array([30.0]))[0] - 30.0) < 1e-12


def test_tau_embedding_closed_forms():
    e0 = O.tau_embedding(0.0, 8)
    assert e0.tolist() == [0, 0, 0, 0, 1, 1, 1, 1]
    e = O.tau_embedding(0.37, 8)
    # w = 10000^(-2i/8) = 1, 0.1, 0.01, 0.001
    for i, w in enumerate([1.0, 0.1, 0.01, 0.001]):
        assert abs(e[i] - math.sin(370.0 * w)) < 1e-12
        assert abs(e[i + 4] - math.cos(370.0 * w)) < 1e-12


def test_linear_orientation_brute_force():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((3, 5))
    w = rng.standard_normal((4, 5))        # [out][in]
    y = O.linear(x, w)
    assert y.shape == (3, 4)
    for r in range(3):
        np.testing.assert_allclose(y[r], BF.matvec_out_in(w.tolist(), x[r].tolist()), atol=1e-14)


# --------------------------------------------------------------------------
# K/V cache
# --------------------------------------------------------------------------

def _slices(rng, L, units, T, H, D):
    return rng.standard_normal((L, units * T, H, D)), rng.standard_normal((L, units * T, H, D))


def test_cache_unit_by_unit_equals_bulk():
    rng = np.random.default_rng(10)
    k, v = _slices(rng, 2, 3, 4, 2, 3)
    a = O.KVCache(2, 5, 4, 2, 3)
    for u in range(3):
        assert a.append(k[:, u * 4:(u + 1) * 4], v[:, u * 4:(u + 1) * 4])
    b = O.KVCache(2, 5, 4, 2, 3)
    assert b.append(k, v)
    assert np.array_equal(a.k, b.k) and np.array_equal(a.v, b.v)
    assert a.units == b.units == 3 and a.valid_tokens == 12 and a.tokens_appended == 12
    assert np.array_equal(a.k[:, :12], k) and np.all(a.k[:, 12:] == 0)


def test_cache_ring_wrap_overwrites_oldest_slot_only():
    rng = np.random.default_rng(11)
    k, v = _slices(rng, 1, 4, 2, 1, 2)
    c = O.KVCache(1, 3, 2, 1, 2, ring=True)
    assert c.append(k[:, :6], v[:, :6])
    before = c.k.copy()
    assert c.append(k[:, 6:8], v[:, 6:8])
    assert np.array_equal(c.k[:, 0:2], k[:, 6:8])          # slot 0 <- unit 3
    assert np.array_equal(c.k[:, 2:6], before[:, 2:6])     # other slots untouched
    assert c.units == 4 and c.valid_tokens == 6 and c.tokens_appended == 8


def test_cache_full_without_ring_refuses_and_keeps_contents():
    rng = np.random.default_rng(12)
    k, v = _slices(rng, 1, 3, 2, 1, 2)
    c = O.KVCache(1, 2, 2, 1, 2, ring=False)
    assert c.append(k[:, :4], v[:, :4])
    snap = c.k.copy(), c.v.copy()
    assert not c.append(k[:, 4:6], v[:, 4:6])
    assert np.array_equal(c.k, snap[0]) and np.array_equal(c.v, snap[1]) and c.units == 2
    with pytest.raises(ValueError):
        c.append(k[:, :3], v[:, :3])


# --------------------------------------------------------------------------
# the velocity network
# --------------------------------------------------------------------------

def _tiny_problem(seed=13, **kw):
    cfg = tiny_cfg(**kw)
    rng = np.random.default_rng(seed)
    w = tiny_weights(cfg, rng)
    S = 6
    ck = [rng.standard_normal((S + 3, cfg.n_heads, cfg.head_dim)) for _ in range(cfg.n_layers)]
    cv = [rng.standard_normal((S + 3, cfg.n_heads, cfg.head_dim)) for _ in range(cfg.n_layers)]
    z = rng.standard_normal((cfg.n_tokens, cfg.c_lat))
    return cfg, w, ck, cv, z, S


def test_f_theta_matches_scalar_brute_force():
    cfg, w, ck, cv, z, S = _tiny_problem()
    got = O.f_theta(cfg, z, 0.75, w, ck, cv, S, 11)
    ref = BF.velocity(cfg, z, 0.75, w, ck, cv, S, 11)
    np.testing.assert_allclose(got, np.array(ref), rtol=1e-11, atol=1e-12)


def test_f_theta_ignores_cache_rows_beyond_valid():
    cfg, w, ck, cv, z, S = _tiny_problem(14)
    a = O.f_theta(cfg, z, 0.5, w, ck, cv, S, 0)
    ck2 = [c.copy() for c in ck]; cv2 = [c.copy() for c in cv]
    for c in ck2 + cv2:
        c[S:] = 1e3
    assert np.array_equal(a, O.f_theta(cfg, z, 0.5, w, ck2, cv2, S, 0))
    ck2[0][S - 1] += 1.0
    assert not np.array_equal(a, O.f_theta(cfg, z, 0.5, w, ck2, cv2, S, 0))


def test_f_theta_in_unit_permutation_equivariance():
    cfg, w, ck, cv, z, S = _tiny_problem(15)
    n = cfg.n_tokens
    pos = 20 + np.arange(n)
    mod = O.modality_of_tokens(cfg)
    perm = np.random.default_rng(0).permutation(n)
    a = O.f_theta(cfg, z, 0.25, w, ck, cv, S, 20)
    b = O.f_theta(cfg, z[perm], 0.25, w, ck, cv, S, 20, pos=pos[perm], modality=mod[perm])
    np.testing.assert_allclose(b, a[perm], atol=1e-12)


def test_f_theta_cross_modal_coupling():
    cfg, w, ck, cv, z, S = _tiny_problem(16)
    a = O.f_theta(cfg, z, 1.0, w, ck, cv, S, 5)
    za = z.copy(); za[cfg.n_video] += 1.0            # perturb one audio token
    b = O.f_theta(cfg, za, 1.0, w, ck, cv, S, 5)
    assert np.max(np.abs(b[:cfg.n_video] - a[:cfg.n_video])) > 1e-6
    zv = z.copy(); zv[0] += 1.0                      # perturb one video token
    c = O.f_theta(cfg, zv, 1.0, w, ck, cv, S, 5)
    assert np.max(np.abs(c[cfg.n_video:] - a[cfg.n_video:])) > 1e-6


def test_block_causal_sequence_future_units_do_not_leak():
    cfg = tiny_cfg()
    rng = np.random.default_rng(17)
    w = tiny_weights(cfg, rng)
    zs = [rng.standard_normal((cfg.n_tokens, cfg.c_lat)) for _ in range(4)]
    taus = [0.0, 0.0, 0.5, 1.0]
    base = O.f_theta_sequence(cfg, zs, taus, w)
    zs2 = list(zs); zs2[3] = zs[3] + 5.0            # perturb the last unit only
    pert = O.f_theta_sequence(cfg, zs2, taus, w)
    for u in range(3):
        assert np.array_equal(base[u], pert[u])
    assert not np.array_equal(base[3], pert[3])


def test_performer_form_equals_block_causal_sequence():
    # The performer's cache holds the rotated K/V of earlier units; attending to it
    # plus the whole current unit must reproduce the masked full-sequence output.
    cfg = tiny_cfg(unit_kv_tokens=5)                 # a cached unit = one unit of tokens
    rng = np.random.default_rng(18)
    w = tiny_weights(cfg, rng)
    n_units = 4
    zs = [rng.standard_normal((cfg.n_tokens, cfg.c_lat)) for _ in range(n_units)]
    taus = [0.0, 0.0, 0.0, 0.6]
    seq, kv = O.f_theta_sequence(cfg, zs, taus, w, return_kv=True)
    n = cfg.n_tokens
    cache = O.KVCache(cfg.n_layers, 8, n, cfg.n_heads, cfg.head_dim)
    for u in range(n_units - 1):
        cache.append(np.stack([kv[l][0][u * n:(u + 1) * n] for l in range(cfg.n_layers)]),
                     np.stack([kv[l][1][u * n:(u + 1) * n] for l in range(cfg.n_layers)]))
    got = O.f_theta(cfg, zs[-1], taus[-1], w, cache.k, cache.v, cache.valid_tokens,
                    cache.tokens_appended)
    np.testing.assert_allclose(got, seq[-1], atol=1e-12)


def _units_problem(seed, n_units=3, S=10):
    cfg = tiny_cfg(unit_kv_tokens=5)
    rng = np.random.default_rng(seed)
    w = tiny_weights(cfg, rng)
    ck = [rng.standard_normal((S + 4, cfg.n_heads, cfg.head_dim)) for _ in range(cfg.n_layers)]
    cv = [rng.standard_normal((S + 4, cfg.n_heads, cfg.head_dim)) for _ in range(cfg.n_layers)]
    zs = [rng.standard_normal((cfg.n_tokens, cfg.c_lat)) for _ in range(n_units)]
    return cfg, w, ck, cv, zs, S


def test_units_pass_with_empty_prefix_is_the_block_causal_sequence():
    cfg, w, ck, cv, zs, _ = _units_problem(40)
    taus = [0.0, 0.3, 1.0]
    seq, kv_seq = O.f_theta_sequence(cfg, zs, taus, w, return_kv=True)
    got, kv = O.f_theta_units(cfg, zs, taus, w, ck, cv, 0, 0, return_kv=True)
    for a, b in zip(got, seq):
        np.testing.assert_allclose(a, b, atol=1e-12)
    for (k1, v1), (k2, v2) in zip(kv, kv_seq):
        np.testing.assert_allclose(k1, k2, atol=1e-12)
        np.testing.assert_allclose(v1, v2, atol=1e-12)


def test_units_pass_of_one_unit_is_f_theta():
    cfg, w, ck, cv, zs, S = _units_problem(41, n_units=1)
    got = O.f_theta_units(cfg, zs, [0.7], w, ck, cv, S, 37)[0]
    np.testing.assert_allclose(got, O.f_theta(cfg, zs[0], 0.7, w, ck, cv, S, 37), atol=1e-12)
    # and the brute-force scalar loops agree
    np.testing.assert_allclose(got, np.array(BF.velocity(cfg, zs[0], 0.7, w, ck, cv, S, 37)),
                               rtol=1e-11, atol=1e-12)


def test_units_pass_equals_performer_form_over_the_grown_cache():
    # unit u of the pass sees the prefix and units < u: the performer form with those
    # units' own K/V appended to the cache (positions continuing) gives the same result
    cfg, w, ck, cv, zs, S = _units_problem(42, n_units=3)
    taus = [0.0, 0.25, 0.9]
    p0 = 19
    got, kv = O.f_theta_units(cfg, zs, taus, w, ck, cv, S, p0, return_kv=True)
    n = cfg.n_tokens
    for u in range(3):
        gk = [np.concatenate([ck[l][:S], kv[l][0][:u * n]]) for l in range(cfg.n_layers)]
        gv = [np.concatenate([cv[l][:S], kv[l][1][:u * n]]) for l in range(cfg.n_layers)]
        ref = O.f_theta(cfg, zs[u], taus[u], w, gk, gv, S + u * n, p0 + u * n)
        np.testing.assert_allclose(got[u], ref, atol=1e-12)


def test_units_pass_later_units_do_not_leak_and_prefix_matters():
    cfg, w, ck, cv, zs, S = _units_problem(43, n_units=3)
    taus = [0.5, 0.5, 0.5]
    base = O.f_theta_units(cfg, zs, taus, w, ck, cv, S, 3)
    zs2 = list(zs); zs2[2] = zs[2] + 4.0
    pert = O.f_theta_units(cfg, zs2, taus, w, ck, cv, S, 3)
    assert np.array_equal(base[0], pert[0]) and np.array_equal(base[1], pert[1])
    assert not np.array_equal(base[2], pert[2])
    ck2 = [c.copy() for c in ck]
    ck2[1][0] += 1.0                                  # a cached key every unit sees
    moved = O.f_theta_units(cfg, zs, taus, w, ck2, cv, S, 3)
    assert all(np.max(np.abs(m - b)) > 1e-9 for m, b in zip(moved, base))


def test_solve_with_network_is_euler_over_f_theta():
    cfg, w, ck, cv, z, S = _tiny_problem(19)
    taus = [1.0, 0.5, 0.0]
    got = O.denoise_solve(cfg, z, taus, w, ck, cv, S, 3)
    v1 = np.array(BF.velocity(cfg, z, 1.0, w, ck, cv, S, 3))
    z1 = z - 0.5 * v1
    v2 = np.array(BF.velocity(cfg, z1, 0.5, w, ck, cv, S, 3))
    np.testing.assert_allclose(got, z1 - 0.5 * v2, rtol=1e-11, atol=1e-12)


def test_step_flops_counts():
    cfg = O.Config(28, 3072, 24, 128, 12288, 16, 920, 4, 1200)
    f = O.step_flops(cfg, 57600)
    attn = 4 * 924 * (57600 + 924) * 3072
    assert abs(attn / 28 / 1e9 * 28 - attn / 1e9) < 1e-9
    assert abs(f / 1e12 - 24.47) < 0.01          # per Euler step at the 640x368 unit


# --------------------------------------------------------------------------
# classifier-free guidance
# --------------------------------------------------------------------------

def test_guided_velocity_closed_form_with_exact_fields():
    # Constant fields aiming at two clean latents a (conditional) and b
    # (unconditional): one Euler step 1 -> 0 from eps lands on b + s (a - b), so
    # s = 0, 1 give b and a, and s = 3 extrapolates three times past b.
    rng = np.random.default_rng(40)
    a, b, eps = (rng.standard_normal((5, 3)) for _ in range(3))
    for s in (0.0, 1.0, 3.0, -0.5):
        v = O.guided_velocity(O.rf_velocity(a, eps), O.rf_velocity(b, eps), s)
        got = O.fm_solve(eps, [1.0, 0.0], lambda z, t, v=v: v)
        np.testing.assert_allclose(got, b + s * (a - b), rtol=0, atol=1e-14)


def _cfg_problem(seed):
    cfg, w, ck, cv, z, S = _tiny_problem(seed)
    rng = np.random.default_rng(seed + 100)
    uk = [rng.standard_normal(c.shape) for c in ck]
    uv = [rng.standard_normal(c.shape) for c in cv]
    return cfg, w, z, (ck, cv, S, 7), (uk, uv, 2, 0)


def test_guided_solve_scale_one_is_conditional_and_zero_is_unconditional():
    cfg, w, z, cond, uncond = _cfg_problem(41)
    taus = [1.0, 0.6, 0.2, 0.0]
    c = O.denoise_solve(cfg, z, taus, w, *cond)
    u = O.denoise_solve(cfg, z, taus, w, *uncond)
    assert np.max(np.abs(c - u)) > 1e-3                 # the two contexts differ
    np.testing.assert_allclose(O.denoise_solve_cfg(cfg, z, taus, w, cond, uncond, 1.0), c,
                               rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.denoise_solve_cfg(cfg, z, taus, w, cond, uncond, 0.0), u,
                               rtol=0, atol=1e-12)


def test_guided_solve_with_equal_contexts_ignores_the_scale():
    cfg, w, z, cond, _ = _cfg_problem(42)
    taus = [1.0, 0.5, 0.0]
    plain = O.denoise_solve(cfg, z, taus, w, *cond)
    for s in (0.0, 2.5, 7.0):
        np.testing.assert_allclose(O.denoise_solve_cfg(cfg, z, taus, w, cond, cond, s), plain,
                                   rtol=0, atol=1e-11)


def test_guided_solve_matches_brute_force_velocities():
    # Two Euler steps with the scalar-loop velocity network on each context.
    cfg, w, z, cond, uncond = _cfg_problem(43)
    s = 4.0
    got = O.denoise_solve_cfg(cfg, z, [1.0, 0.5, 0.0], w, cond, uncond, s)
    zz = z
    for t in (1.0, 0.5):
        vc = np.array(BF.velocity(cfg, zz, t, w, *cond))
        vu = np.array(BF.velocity(cfg, zz, t, w, *uncond))
        zz = zz - 0.5 * (vu + s * (vc - vu))
    np.testing.assert_allclose(got, zz, rtol=1e-10, atol=1e-11)


# --------------------------------------------------------------------------
# open-reading variants: 3-D rotary embedding, SwiGLU MLP, 64-channel tokens
# --------------------------------------------------------------------------

def test_rope_3d_scalar_brute_force():
    # D = 12: 6 rotate-half pairs, 2 per axis (t, y, x); pair k of an axis turns by
    # pos_axis * theta^(-k / 2)
    rng = np.random.default_rng(50)
    x = rng.standard_normal((3, 2, 12))
    pos3 = np.array([[3, 1, 2], [0, 4, 1], [7, 0, 0]])
    theta = 100.0
    got = O.rope_3d(x, pos3, theta)
    assert O.rope_3d_bands(12) == (2, 2, 2)
    for n in range(3):
        for h in range(2):
            for i in range(6):
                ax, k = i // 2, i % 2
                ang = pos3[n, ax] * theta ** (-k / 2.0)
                a, b = x[n, h, i], x[n, h, i + 6]
                assert abs(got[n, h, i] - (a * math.cos(ang) - b * math.sin(ang))) < 1e-12
                assert abs(got[n, h, i + 6] - (b * math.cos(ang) + a * math.sin(ang))) < 1e-12


def test_rope_3d_bands_and_relative_positions():
    assert O.rope_3d_bands(128) == (22, 21, 21)        # the Wan split of 64 pairs
    assert O.rope_3d_bands(64) == (12, 10, 10)
    rng = np.random.default_rng(51)
    q = rng.standard_normal((1, 1, 128))
    k = rng.standard_normal((1, 1, 128))
    def dot(a, b):
        return float((O.rope_3d(q, [a], 1e4) * O.rope_3d(k, [b], 1e4)).sum())
    # depends on the position differences only, per axis
    assert abs(dot((5, 2, 7), (3, 1, 1)) - dot((12, 6, 9), (10, 5, 3))) < 1e-9
    assert abs(dot((5, 2, 7), (3, 1, 1)) - dot((5, 2, 7), (3, 2, 1))) > 1e-6
    # rotations keep every pair's norm; (0, 0, 0) is the identity
    y = O.rope_3d(q, [(9, 4, 33)], 1e4)
    np.testing.assert_allclose(y[..., :64] ** 2 + y[..., 64:] ** 2, q[..., :64] ** 2 + q[..., 64:] ** 2,
                               atol=1e-12)
    np.testing.assert_array_equal(O.rope_3d(q, [(0, 0, 0)], 1e4), q)


def test_token_positions_3d_raster_and_audio():
    cfg = tiny_cfg(n_video=6, n_audio=2, unit_kv_tokens=8)
    cfg.rope_mode, cfg.grid_w = "3d", 3
    pos = O.token_positions(cfg, 16, n_units=2)           # p0 = 16 tokens = 2 units
    assert pos.shape == (16, 3)
    np.testing.assert_array_equal(pos[:8], [[2, 0, 0], [2, 0, 1], [2, 0, 2], [2, 1, 0], [2, 1, 1],
                                            [2, 1, 2], [2, 0, 0], [2, 0, 0]])
    np.testing.assert_array_equal(pos[8:, 0], [3] * 8)
    cfg.rope_mode = "1d"
    np.testing.assert_array_equal(O.token_positions(cfg, 16, n_units=2), 16 + np.arange(16))


def test_silu_and_swiglu_layout():
    x = np.linspace(-30, 30, 121)
    np.testing.assert_allclose(O.silu(x), x * scipy.special.expit(x), rtol=1e-13, atol=1e-15)
    assert O.silu(0.0) == 0.0 and abs(O.silu(40.0) - 40.0) < 1e-12
    rng = np.random.default_rng(52)
    wg = rng.standard_normal((128, 5))
    wu = rng.standard_normal((128, 5))
    w1 = np.concatenate([np.concatenate([wg[64 * b:64 * b + 64], wu[64 * b:64 * b + 64]]) for b in range(2)])
    g, u = O.swiglu_gate_up(None, w1)
    np.testing.assert_array_equal(g, wg)
    np.testing.assert_array_equal(u, wu)


def test_swiglu_mlp_brute_force():
    cfg = tiny_cfg(d_mlp=64)
    cfg.mlp = "swiglu"
    rng = np.random.default_rng(53)
    h = rng.standard_normal((3, cfg.d_model))
    lw = {"w_1": rng.standard_normal((128, cfg.d_model)) * 0.3,
          "w_2": rng.standard_normal((cfg.d_model, 64)) * 0.3}
    got = O.mlp_forward(cfg, h, lw)
    for r in range(3):
        for o in range(cfg.d_model):
            acc = 0.0
            for f in range(64):
                g = sum(h[r, c] * lw["w_1"][f, c] for c in range(cfg.d_model))        # gate rows 0..63
                u = sum(h[r, c] * lw["w_1"][64 + f, c] for c in range(cfg.d_model))   # up rows 64..127
                acc += g / (1.0 + math.exp(-g)) * u * lw["w_2"][o, f]
            assert abs(got[r, o] - acc) < 1e-10


@pytest.mark.parametrize("mlp,rope_mode", [("swiglu", "1d"), ("gelu", "3d"), ("swiglu", "3d")])
def test_variant_performer_form_equals_block_causal_sequence(mlp, rope_mode):
    # the performer form over a cache of earlier units' own K/V equals the masked
    # full-sequence form with the variant MLP and rotary embedding too
    cfg = tiny_cfg(unit_kv_tokens=5, d_mlp=64)
    cfg.mlp, cfg.rope_mode, cfg.grid_w = mlp, rope_mode, 3
    rng = np.random.default_rng(54)
    w = tiny_weights(cfg, rng)
    if mlp == "swiglu":
        for lw in w["layers"]:
            lw["w_1"] = rng.standard_normal((2 * cfg.d_mlp, cfg.d_model)) * 0.3
    zs = [rng.standard_normal((cfg.n_tokens, cfg.c_lat)) for _ in range(3)]
    taus = [0.0, 0.0, 0.6]
    seq, kv = O.f_theta_sequence(cfg, zs, taus, w, return_kv=True)
    n = cfg.n_tokens
    ck = [kv[l][0][:2 * n] for l in range(cfg.n_layers)]
    cv = [kv[l][1][:2 * n] for l in range(cfg.n_layers)]
    got = O.f_theta(cfg, zs[2], taus[2], w, ck, cv, 2 * n, 2 * n)
    np.testing.assert_allclose(got, seq[2], atol=1e-12)
    units = O.f_theta_units(cfg, zs, taus, w, ck, cv, 0, 0)
    for a, b in zip(units, seq):
        np.testing.assert_allclose(a, b, atol=1e-12)
    # the variant changes the result (it is not silently ignored)
    cfg2 = tiny_cfg(unit_kv_tokens=5, d_mlp=64)
    if mlp == "gelu":
        assert np.max(np.abs(O.f_theta_sequence(cfg2, zs, taus, w)[2] - seq[2])) > 1e-6
