"""K/V cache writer through the C ABI: bit-exact against the oracle's ring
cache, host-side error paths, and the full-size append."""
import numpy as np
import pytest
import torch

import sfm_synth as S
from oracle import sfm_oracle as O
from streaming_flow_matching_b200 import _lib as L

pytestmark = pytest.mark.gpu

W = S.Workload("cache-small", 3, 256, 4, 128, 512, 16, 10, 2, 7, 3, 1, "bf16")


def _perf(w, cache_units, ring=True, sessions=1):
    from streaming_flow_matching_b200 import Performer
    pool = sessions * (cache_units * w.unit_kv_tokens + w.n_tokens)
    return Performer.from_workload(w.replace(cache_units=cache_units), None, pool_tokens=pool,
                                   max_sessions=sessions, ring=ring)


def _read_all(p, s, w, cache_units):
    rows = cache_units * w.unit_kv_tokens
    ks, vs = zip(*[p.kvcache_read(s, l, 0, rows) for l in range(w.n_layers)])
    return torch.stack(ks).cpu(), torch.stack(vs).cpu()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_append_unit_by_unit_and_bulk_match_oracle_ring(cuda_device, dtype):
    w = W.replace(dtype=dtype) if dtype == "bf16" else W.replace(dtype=dtype, head_dim=64)
    n_units, cap = 5, 3
    k, v = S.make_kv_slices(w, n_units)
    ref = O.KVCache(w.n_layers, cap, w.unit_kv_tokens, w.n_heads, w.head_dim)
    ref.append(O.f64(k), O.f64(v))
    p = _perf(w, cap, sessions=2)
    a = p.open_session(cap)
    b = p.open_session(cap)
    T = w.unit_kv_tokens
    for u in range(n_units):
        p.kvcache_append(a, k[:, u * T:(u + 1) * T].contiguous().cuda(),
                         v[:, u * T:(u + 1) * T].contiguous().cuda())
    p.kvcache_append(b, k.cuda(), v.cuda())            # bulk: 5 units into 3 slots
    torch.cuda.synchronize()
    for s in (a, b):
        gk, gv = _read_all(p, s, w, cap)
        assert np.array_equal(O.f64(gk), ref.k) and np.array_equal(O.f64(gv), ref.v)
        info = p.session_info(s)
        assert info["units_appended"] == 5 and info["valid_tokens"] == 3 * T and info["p0"] == 5 * T
    p.close()


def test_ring_off_refuses_when_full_and_keeps_contents(cuda_device):
    w = W
    k, v = S.make_kv_slices(w, 3)
    p = _perf(w, 2, ring=False)
    s = p.open_session(2)
    T = w.unit_kv_tokens
    p.kvcache_append(s, k[:, :2 * T].contiguous().cuda(), v[:, :2 * T].contiguous().cuda())
    torch.cuda.synchronize()
    before = _read_all(p, s, w, 2)
    with pytest.raises(L.SfmError) as e:
        p.kvcache_append(s, k[:, 2 * T:].contiguous().cuda(), v[:, 2 * T:].contiguous().cuda())
    assert e.value.status == L.SFM_ECAPACITY
    after = _read_all(p, s, w, 2)
    assert torch.equal(before[0], after[0]) and torch.equal(before[1], after[1])
    assert p.session_info(s)["units_appended"] == 2
    p.close()


def test_host_errors_on_a_live_handle(cuda_device):
    w = W
    p = _perf(w, 2)
    s = p.open_session(2)
    k, v = S.make_kv_slices(w, 1)
    kc, vc = k.cuda(), v.cuda()
    h = p._h
    st = torch.cuda.current_stream().cuda_stream
    import ctypes as C
    assert L.lib.sfm_kvcache_append(h, 5, C.c_void_p(kc.data_ptr()), C.c_void_p(vc.data_ptr()), 7, C.c_void_p(st)) == L.SFM_ESESSION
    assert L.lib.sfm_kvcache_append(h, s, C.c_void_p(kc.data_ptr()), C.c_void_p(vc.data_ptr()), 6, C.c_void_p(st)) == L.SFM_EINVAL
    assert L.lib.sfm_kvcache_append(h, s, C.c_void_p(kc.data_ptr() + 2), C.c_void_p(vc.data_ptr()), 7, C.c_void_p(st)) == L.SFM_EINVAL
    assert L.lib.sfm_kvcache_read(h, s, 3, 0, 1, C.c_void_p(kc.data_ptr()), C.c_void_p(vc.data_ptr()), C.c_void_p(st)) == L.SFM_EINVAL
    assert L.lib.sfm_kvcache_read(h, s, 0, 0, 100, C.c_void_p(kc.data_ptr()), C.c_void_p(vc.data_ptr()), C.c_void_p(st)) == L.SFM_EINVAL
    z = torch.zeros(w.n_tokens, w.c_lat, device="cuda")
    assert L.lib.sfm_denoise_step(h, s, C.c_void_p(z.data_ptr()), 1.0, 0.5, None, C.c_void_p(st)) == L.SFM_EINVAL  # no weights
    out = C.c_int()
    assert L.lib.sfm_session_open(h, 2, C.byref(out)) == L.SFM_ECAPACITY   # table full
    assert p.session_info(s)["units_appended"] == 0
    p.close()


def test_full_size_append_wraps_into_slot_zero(cuda_device):
    # 640x368: 48 units cached, one more 1200-token slice evicts unit 0 (slot 0)
    w = S.V02
    from streaming_flow_matching_b200 import Performer
    p = Performer.from_workload(w, None)
    s = p.open_session(w.cache_units)
    k, v = S.make_kv_slices(w, w.cache_units, device="cuda")
    p.kvcache_append(s, k, v)
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    shape = (w.n_layers, w.unit_kv_tokens, w.n_heads, w.head_dim)
    k1 = torch.randn(*shape, generator=g, device="cuda").to(torch.bfloat16)
    v1 = torch.randn(*shape, generator=g, device="cuda").to(torch.bfloat16)
    p.kvcache_append(s, k1, v1)
    torch.cuda.synchronize()
    T = w.unit_kv_tokens
    for layer in (0, 13, 27):
        gk, gv = p.kvcache_read(s, layer, 0, 2 * T)
        assert torch.equal(gk[:T], k1[layer]) and torch.equal(gv[:T], v1[layer])
        assert torch.equal(gk[T:], k[layer, T:2 * T]) and torch.equal(gv[T:], v[layer, T:2 * T])
        gk, gv = p.kvcache_read(s, layer, 47 * T, T)
        assert torch.equal(gk, k[layer, 47 * T:]) and torch.equal(gv, v[layer, 47 * T:])
    info = p.session_info(s)
    assert info["units_appended"] == 49 and info["valid_tokens"] == 57600 and info["p0"] == 49 * T
    p.close()


@pytest.mark.parametrize("world", [2, 4])
def test_head_sharded_append_takes_each_ranks_head_range(cuda_device, world):
    # each rank of a head-sharded cache (Ulysses group of `world` ranks) keeps heads
    # [r H / P, (r + 1) H / P) of the broadcast slice, bit for bit, ring included
    from streaming_flow_matching_b200.ulysses import UlyssesPlan, cache_heads
    w = W.replace(n_heads=4)
    n_units, cap = 5, 3
    k, v = S.make_kv_slices(w, n_units)
    plan = UlyssesPlan(w.n_video, w.n_audio, w.n_heads, world)
    for r in range(world):
        wr = w.replace(n_heads=plan.heads_per_rank)
        ref = O.KVCache(w.n_layers, cap, w.unit_kv_tokens, wr.n_heads, w.head_dim)
        ref.append(O.f64(cache_heads(plan, k, r)), O.f64(cache_heads(plan, v, r)))
        p = _perf(wr, cap)
        s = p.open_session(cap)
        h0, _ = plan.head_range(r)
        p.kvcache_append_heads(s, k.cuda(), v.cuda(), h0)
        torch.cuda.synchronize()
        gk, gv = _read_all(p, s, wr, cap)
        assert np.array_equal(O.f64(gk), ref.k) and np.array_equal(O.f64(gv), ref.v)
        assert p.session_info(s)["units_appended"] == n_units
        # a head range past the slice's heads is refused before any launch
        with pytest.raises(Exception):
            p.kvcache_append_heads(s, k.cuda(), v.cuda(), w.n_heads - plan.heads_per_rank + 1)
        p.close()
