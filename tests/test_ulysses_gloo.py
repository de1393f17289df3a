"""Ulysses context parallelism of the performer on CPU with gloo ranks: each rank
owns a shard of the video tokens plus every audio token and a group of heads;
one f_theta layer run through the module's all-to-alls (the per-rank arithmetic
taken from the oracle) must equal the oracle's unsharded layer on every rank's
rows, and the gathered velocities must equal the unsharded head.  Ragged video
shards (7 tokens over 2 and 4 ranks) and replicated audio are covered."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    from oracle import sfm_oracle as O
    cfg = O.Config(n_layers=1, d_model=16, n_heads=4, head_dim=4, d_mlp=32, c_lat=3, n_video=7,
                   n_audio=2, unit_kv_tokens=5)
    rng = np.random.default_rng(90)
    n = lambda *s: rng.standard_normal(s) * 0.3
    w = {"w_in": n(cfg.d_model, cfg.c_lat), "e_mod": n(2, cfg.d_model),
         "g_final": 1.0 + 0.1 * rng.standard_normal(cfg.d_model), "w_out": n(cfg.c_lat, cfg.d_model),
         "layers": [{"g_attn": 1.0 + 0.1 * rng.standard_normal(cfg.d_model),
                     "w_qkv": n(3 * cfg.hd, cfg.d_model), "w_o": n(cfg.d_model, cfg.hd),
                     "g_mlp": 1.0 + 0.1 * rng.standard_normal(cfg.d_model),
                     "w_1": n(cfg.d_mlp, cfg.d_model), "w_2": n(cfg.d_model, cfg.d_mlp)}]}
    S = 10
    ck = rng.standard_normal((S, cfg.n_heads, cfg.head_dim))
    cv = rng.standard_normal((S, cfg.n_heads, cfg.head_dim))
    z = rng.standard_normal((cfg.n_tokens, cfg.c_lat))
    return cfg, w, ck, cv, z, S


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from oracle import sfm_oracle as O
        from streaming_flow_matching_b200 import ulysses as U
        cfg, w, ck, cv, z, S = _problem()
        plan = U.UlyssesPlan(cfg.n_video, cfg.n_audio, cfg.n_heads, world)
        tau, p0 = 0.6, 40
        lw = w["layers"][0]
        loc = plan.local_tokens(rank)
        H, D = cfg.n_heads, cfg.head_dim
        # the rank's own rows through one layer; attention over its head group
        x = O.embed(cfg, z, tau, w)[loc]
        h = O.rmsnorm(x, lw["g_attn"], cfg.rms_eps)
        qkv = O.linear(h, lw["w_qkv"])
        nl = len(loc)
        q = qkv[:, :cfg.hd].reshape(nl, H, D)
        k = qkv[:, cfg.hd:2 * cfg.hd].reshape(nl, H, D)
        v = qkv[:, 2 * cfg.hd:].reshape(nl, H, D)
        pos = p0 + np.array(loc)
        q, k = O.rope(q, pos, cfg.rope_theta), O.rope(k, pos, cfg.rope_theta)
        qh, kh, vh = (U.seq_to_heads(plan, torch.from_numpy(t), rank).numpy() for t in (q, k, v))
        kc = U.cache_heads(plan, torch.from_numpy(ck), rank).numpy()
        vc = U.cache_heads(plan, torch.from_numpy(cv), rank).numpy()
        a = O.attention(qh, np.concatenate([kc, kh]), np.concatenate([vc, vh]))
        o = U.heads_to_seq(plan, torch.from_numpy(a), rank).numpy()
        x = x + O.linear(o.reshape(nl, cfg.hd), lw["w_o"])
        h2 = O.rmsnorm(x, lw["g_mlp"], cfg.rms_eps)
        x = x + O.linear(O.gelu_tanh(O.linear(h2, lw["w_1"])), lw["w_2"])
        vel = U.gather_latents(plan, torch.from_numpy(O.head(cfg, x, w)), rank).numpy()
        # the unsharded reference
        x_ref = O.layer_forward(cfg, O.embed(cfg, z, tau, w), lw, ck, cv, p0 + np.arange(cfg.n_tokens))
        out_q.put((rank, float(np.max(np.abs(x - x_ref[loc]))),
               float(np.max(np.abs(vel - O.head(cfg, x_ref, w)))), plan.n_video_local(rank)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_layer_equals_unsharded_oracle_layer(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sum(g[3] for g in got) == 7                 # the shards cover the video tokens
    for rank, e_x, e_v, _ in got:
        assert e_x < 1e-12, (rank, e_x)
        assert e_v < 1e-12, (rank, e_v)


def test_plan_index_maps():
    from streaming_flow_matching_b200.ulysses import UlyssesPlan
    p = UlyssesPlan(n_video=920, n_audio=4, n_heads=24, world=8)
    assert [p.n_video_local(r) for r in range(8)] == [115] * 8
    assert p.head_range(3) == (9, 12) and p.heads_per_rank == 3
    assert p.local_tokens(7)[:2] == [805, 806] and p.local_tokens(7)[-4:] == [920, 921, 922, 923]
    r = UlyssesPlan(n_video=7, n_audio=2, n_heads=4, world=4)
    assert [r.video_range(i) for i in range(4)] == [(0, 1), (1, 3), (3, 5), (5, 7)]
    covered = sorted(t for i in range(4) for t in r.local_tokens(i) if t < 7)
    assert covered == list(range(7))
    with pytest.raises(ValueError):
        UlyssesPlan(n_video=920, n_audio=4, n_heads=24, world=5)
