"""Seeded inputs are deterministic and shaped as the workloads state; the oracle
reproduces its committed regression fixture."""
import json
import os

import numpy as np
import torch

import sfm_synth as S
from tests.golden import make_golden


def test_workload_shapes_follow_the_unit_sizes():
    # 640x368 unit -> 40 x 23 video tokens + 4 audio; 192x336 -> 12 x 21 + 4
    assert S.V02.n_video == 40 * 23 and S.V02.n_tokens == 924
    assert S.V01.n_video == 12 * 21 and S.V01.n_tokens == 256
    assert S.V02.cache_units * S.V02.unit_kv_tokens == 57600
    assert S.TINY.n_tokens == 68 and S.TINY.cache_units * S.TINY.unit_kv_tokens == 384


def test_weights_deterministic_and_scaled():
    a = S.make_weights(S.TINY)
    b = S.make_weights(S.TINY)
    assert torch.equal(a["layers"][1]["w_1"], b["layers"][1]["w_1"])
    w = a["layers"][0]["w_qkv"]
    assert w.shape == (3 * 256, 256) and w.dtype == torch.float32
    assert abs(w.std().item() - 0.02) < 1e-3
    assert torch.all(a["layers"][0]["g_attn"] == 1)
    bf = S.make_weights(S.TINY.replace(dtype="bf16"))
    assert bf["w_in"].dtype == torch.bfloat16
    # bf16 values are the fp32 draws rounded to nearest even
    assert torch.equal(bf["w_in"], a["w_in"].to(torch.bfloat16))


def test_slices_and_latents():
    k, v = S.make_kv_slices(S.TINY, 3)
    assert k.shape == (2, 3 * 96, 4, 64)
    k2, _ = S.make_kv_slices(S.TINY, 3)
    assert torch.equal(k, k2) and not torch.equal(k, v)
    z0, eps = S.make_latents(S.TINY, n_sessions=2)
    assert z0.shape == (2, 68, 16) and not torch.equal(z0, eps)


def test_session_lengths_ragged_in_range():
    u = S.session_cache_units()
    assert len(u) == 8 and len(set(u)) > 1
    assert all(8192 <= x * 1200 < 65536 + 1200 for x in u)


def test_oracle_reproduces_committed_regression_fixture():
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny_regression.json")
    with open(path) as f:
        gold = json.load(f)
    w, cfg, weights, cache, eps = make_golden.tiny_case()
    from oracle import sfm_oracle as O
    vel = O.f_theta(cfg, eps, 1.0, weights, cache.k, cache.v, cache.valid_tokens, cache.tokens_appended)
    np.testing.assert_allclose(vel[:4], np.array(gold["velocity_tau1_rows0to3"]), rtol=1e-12, atol=1e-13)
    z = O.denoise_solve(cfg, eps, gold["taus"], weights, cache.k, cache.v, cache.valid_tokens,
                        cache.tokens_appended)
    np.testing.assert_allclose(z[:4], np.array(gold["solve_rows0to3"]), rtol=1e-12, atol=1e-13)
    empty = [O.f64(cache.k[0][:0])] * w.n_layers
    zg = O.denoise_solve_cfg(cfg, eps, gold["taus"], weights,
                             (cache.k, cache.v, cache.valid_tokens, cache.tokens_appended),
                             (empty, empty, 0, 0), gold["guided_scale"])
    np.testing.assert_allclose(zg[:4], np.array(gold["guided_solve_rows0to3"]), rtol=1e-12, atol=1e-13)
