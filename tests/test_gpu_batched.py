"""Several sessions with ragged caches solved in one batched call (the
throughput configuration: independent sessions, one pass of the kernels over
all their tokens) against per-session solves and the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import sfm_synth as S
from oracle import sfm_oracle as O
from streaming_flow_matching_b200 import _lib as L
from tests._gpu_util import BF16_TOL, SMALL_BF16, ocfg, oracle_cache_layers, rel_l2, to_cuda

pytestmark = pytest.mark.gpu

CACHE_UNITS = [2, 5, 3]       # ragged: 200, 500 and 300 cached tokens
APPENDED = [2, 7, 3]          # the second session has wrapped its ring


def _setup(w, max_sessions=3):
    from streaming_flow_matching_b200 import Performer
    weights_cpu = S.make_weights(w)
    weights = to_cuda(weights_cpu)
    pool = sum(u * w.unit_kv_tokens + w.n_tokens for u in CACHE_UNITS)
    p = Performer.from_workload(w, weights, pool_tokens=pool, max_sessions=max_sessions)
    sessions, slices = [], []
    for i, (cap, n) in enumerate(zip(CACHE_UNITS, APPENDED)):
        s = p.open_session(cap)
        k, v = S.make_kv_slices(w, n, seed=100 + i)
        p.kvcache_append(s, k.cuda(), v.cuda())
        sessions.append(s)
        slices.append((k, v))
    return weights_cpu, p, sessions, slices


def test_batched_solve_matches_single_sessions_and_oracle(cuda_device):
    w = SMALL_BF16
    weights_cpu, p, sessions, slices = _setup(w)
    _, eps = S.make_latents(w, n_sessions=len(sessions))
    taus = S.uniform_taus(w.n_steps)
    zs = [eps[i].cuda().clone() for i in range(len(sessions))]
    p.fm_solve_batched(sessions, zs, taus)
    singles = []
    for i, s in enumerate(sessions):
        z = eps[i].cuda().clone()
        p.fm_solve(s, z, taus)
        singles.append(z)
    torch.cuda.synchronize()
    assert p.check_device_error() == 0
    for i, s in enumerate(sessions):
        # same kernels, different batch composition: only the split-KV rounding may differ
        assert rel_l2(zs[i].cpu().numpy(), singles[i].cpu().numpy()) <= 2e-3
        info = p.session_info(s)
        k, v = slices[i]
        ck, cv = oracle_cache_layers(k, v, APPENDED[i], w.unit_kv_tokens, CACHE_UNITS[i])
        ref = O.denoise_solve(ocfg(w), eps[i], taus, weights_cpu, ck, cv, info["valid_tokens"],
                              info["p0"])
        e = rel_l2(zs[i].cpu().numpy(), ref)
        print(f"session {i}: cache {info['valid_tokens']} tokens, p0 {info['p0']}: rel L2 {e:.3e}")
        assert e <= BF16_TOL
    p.close()


def test_batched_argument_errors(cuda_device):
    import ctypes as C
    w = SMALL_BF16
    _, p, sessions, _ = _setup(w)
    z = [torch.zeros(w.n_tokens, w.c_lat, device="cuda") for _ in range(4)]
    taus = (C.c_float * 3)(1.0, 0.5, 0.0)
    st = C.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call(ids, n=None):
        n = len(ids) if n is None else n
        arr = (C.c_int * max(1, len(ids)))(*ids)
        zp = (C.c_void_p * 4)(*[t.data_ptr() for t in z])
        return L.lib.sfm_fm_solve_batched(p._h, n, arr, zp, taus, 3, st)

    assert call([sessions[0], sessions[0]]) == L.SFM_EINVAL          # duplicate session
    assert call([sessions[0], 7]) == L.SFM_ESESSION                  # unknown session
    assert call([0, 1, 2, 3], n=4) == L.SFM_ECAPACITY                # more than max_sessions
    assert call([], n=0) == L.SFM_EINVAL
    bad = (C.c_float * 1)(1.0)
    arr = (C.c_int * 1)(sessions[0])
    zp = (C.c_void_p * 1)(z[0].data_ptr())
    assert L.lib.sfm_fm_solve_batched(p._h, 1, arr, zp, bad, 1, st) == L.SFM_EINVAL  # one tau
    # the same latent buffer for two sessions: both Euler updates would write it
    arr2 = (C.c_int * 2)(sessions[0], sessions[1])
    zsame = (C.c_void_p * 2)(z[0].data_ptr(), z[0].data_ptr())
    assert L.lib.sfm_fm_solve_batched(p._h, 2, arr2, zsame, taus, 3, st) == L.SFM_EINVAL
    p.close()


def test_batch_mixing_one_split_and_merged_sessions(cuda_device):
    # caches of 1, 10 and 60 units: the batched attention gives the shortest session
    # one key split (its output written by the attention kernel itself) and the others
    # several, merged afterwards -- each session against its own solve and the oracle
    from streaming_flow_matching_b200 import Performer
    w = SMALL_BF16
    caps = [1, 10, 60]
    plan = L.attention_batch_splits(w.n_tokens, [c * w.unit_kv_tokens + w.n_tokens for c in caps],
                                    w.n_heads, torch.cuda.get_device_properties(0).multi_processor_count)
    assert plan[0] == 1 and plan[2] > 1, plan
    weights_cpu = S.make_weights(w)
    pool = sum(c * w.unit_kv_tokens + w.n_tokens for c in caps)
    p = Performer.from_workload(w, to_cuda(weights_cpu), pool_tokens=pool, max_sessions=3)
    sessions, slices = [], []
    for i, cap in enumerate(caps):
        s = p.open_session(cap)
        k, v = S.make_kv_slices(w, cap, seed=300 + i)
        p.kvcache_append(s, k.cuda(), v.cuda())
        sessions.append(s)
        slices.append((k, v))
    _, eps = S.make_latents(w, n_sessions=len(caps))
    taus = S.uniform_taus(w.n_steps)
    zs = [eps[i].cuda().clone() for i in range(len(caps))]
    p.fm_solve_batched(sessions, zs, taus)
    singles = []
    for i, s in enumerate(sessions):
        z = eps[i].cuda().clone()
        p.fm_solve(s, z, taus)
        singles.append(z)
    torch.cuda.synchronize()
    assert p.check_device_error() == 0
    for i, s in enumerate(sessions):
        assert rel_l2(zs[i].cpu().numpy(), singles[i].cpu().numpy()) <= 2e-3
        info = p.session_info(s)
        k, v = slices[i]
        ref = O.denoise_solve(ocfg(w), eps[i], taus, weights_cpu, [k[l] for l in range(k.shape[0])],
                              [v[l] for l in range(v.shape[0])], info["valid_tokens"], info["p0"])
        e = rel_l2(zs[i].cpu().numpy(), ref)
        print(f"session {i}: {caps[i]} units, {plan[i]} split(s): rel L2 {e:.3e}")
        assert e <= BF16_TOL
    p.close()
