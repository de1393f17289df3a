"""Solves launched as one captured CUDA graph (the default) against direct
launches: bit-identical latents and velocities, across successive units (the
executable graph is updated in place as positions, cache lengths and the ring
slot change), for single and batched sessions."""
import pytest
import torch

import sfm_synth as S
from tests._gpu_util import SMALL_BF16, to_cuda

pytestmark = pytest.mark.gpu


def _run_units(p, s, w, slices, eps, graph):
    p.set_graph_mode(graph)
    p.reset_session(s)
    taus = S.uniform_taus(w.n_steps)
    out = []
    for k, v in slices:
        p.kvcache_append(s, k, v)
        z = eps.clone()
        p.fm_solve(s, z, taus)
        vel = torch.empty_like(z)
        z1 = eps.clone()
        p.denoise_step(s, z1, taus[0], taus[1], vel)
        torch.cuda.synchronize()
        out.append((z.cpu(), z1.cpu(), vel.cpu()))
    return out


def test_graph_solve_matches_direct_launches_across_units(cuda_device):
    from streaming_flow_matching_b200 import Performer
    w = SMALL_BF16
    cap = 3
    weights = to_cuda(S.make_weights(w))
    p = Performer.from_workload(w, weights, pool_tokens=cap * w.unit_kv_tokens + w.n_tokens)
    s = p.open_session(cap)
    k, v = S.make_kv_slices(w, 5)
    T = w.unit_kv_tokens
    # 5 units into 3 slots: the cache fills, then wraps (positions keep counting)
    slices = [(k[:, u * T:(u + 1) * T].contiguous().cuda(), v[:, u * T:(u + 1) * T].contiguous().cuda())
              for u in range(5)]
    _, eps = S.make_latents(w)
    eps = eps[0].cuda()
    direct = _run_units(p, s, w, slices, eps, graph=False)
    graphed = _run_units(p, s, w, slices, eps, graph=True)
    for u, (a, b) in enumerate(zip(direct, graphed)):
        for x, y in zip(a, b):
            assert torch.equal(x, y), f"unit {u}"
    p.check_device_error()
    p.close()


def test_graph_batched_solve_matches_direct_launches(cuda_device):
    from streaming_flow_matching_b200 import Performer
    w = SMALL_BF16
    caps = [2, 4, 3]
    weights = to_cuda(S.make_weights(w))
    pool = sum(c * w.unit_kv_tokens + w.n_tokens for c in caps)
    p = Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=len(caps))
    sessions = []
    for i, c in enumerate(caps):
        s = p.open_session(c)
        k, v = S.make_kv_slices(w.replace(cache_units=c), c, seed=S.SEED_CACHE + 10 * i)
        p.kvcache_append(s, k.cuda(), v.cuda())
        sessions.append(s)
    _, eps = S.make_latents(w, device="cuda", n_sessions=len(caps))
    taus = S.uniform_taus(w.n_steps)
    res = []
    for graph in (False, True, True):
        p.set_graph_mode(graph)
        zs = [eps[i].clone() for i in range(len(caps))]
        p.fm_solve_batched(sessions, zs, taus)
        torch.cuda.synchronize()
        res.append([z.cpu() for z in zs])
    for a, b in zip(res[0], res[1]):
        assert torch.equal(a, b)
    for a, b in zip(res[0], res[2]):
        assert torch.equal(a, b)
    p.check_device_error()
    p.close()


def test_graph_guided_solves_alternating_with_plain_ones_match_direct(cuda_device):
    # plain and guided solves keep separate executable graphs; alternating them
    # must give what direct launches give
    from streaming_flow_matching_b200 import Performer
    w = SMALL_BF16
    weights = to_cuda(S.make_weights(w))
    caps = [3, 1]
    pool = sum(c * w.unit_kv_tokens + w.n_tokens for c in caps)
    p = Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=2)
    s = p.open_session(3)
    u = p.open_session(1)
    k, v = S.make_kv_slices(w, 3)
    p.kvcache_append(s, k.cuda(), v.cuda())
    _, eps = S.make_latents(w)
    eps = eps[0].cuda()
    taus = S.uniform_taus(w.n_steps)
    res = []
    for graph in (False, True):
        p.set_graph_mode(graph)
        out = []
        for scale in (3.0, None, 1.5, None):
            z = eps.clone()
            if scale is None:
                p.fm_solve(s, z, taus)
            else:
                p.fm_solve_guided(s, u, z, taus, scale)
            torch.cuda.synchronize()
            out.append(z.cpu())
        res.append(out)
    for i, (a, b) in enumerate(zip(*res)):
        assert torch.equal(a, b), f"call {i}"
    assert not torch.equal(res[1][0], res[1][2])     # the scale reaches the graph
    p.check_device_error()
    p.close()
